/*
 * FP64 CPU oracle for the routed NVFP4 mixture-of-experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the package entry point's smoke check
 * and the bench's CPU-baseline leg may load this library. It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never calls it.
 *
 * Every function computes the plain definition with every weight decoded exactly
 * (E2M1 code x E4M3 group scale x FP32 tensor scale) and all arithmetic in FP64.
 * See nvfp4_moe_oracle.c for the passages each step follows.
 */
#ifndef NVFP4_MOE_ORACLE_H
#define NVFP4_MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t E, H, I, K;
} orc_dims;

typedef struct {
    const uint8_t *gate_codes, *up_codes;    /* [E][I][H/2] */
    const uint8_t *gate_scales, *up_scales;  /* [E][I][H/16] */
    const float *gate_global, *up_global;    /* [E] */
    const uint8_t *down_codes;               /* [E][H][I/2] */
    const uint8_t *down_scales;              /* [E][H][I/16] */
    const float *down_global;                /* [E] */
} orc_weights;

/* Planted mistakes, used only by negative-control tests. */
enum {
    ORC_PLANT_NONE = 0,
    ORC_PLANT_NIBBLE_ORDER = 1,  /* read element 2c from the high nibble      */
    ORC_PLANT_GROUP_SHIFT = 2,   /* use the next group's scale                 */
    ORC_PLANT_NO_GLOBAL = 3,     /* drop the FP32 tensor scales                */
    ORC_PLANT_SWAP_GATE_UP = 4,  /* apply SiLU to u instead of g               */
    ORC_PLANT_SILU_SIGN = 5,     /* z / (1 + exp(+z))                          */
    ORC_PLANT_EQUAL_WEIGHTS = 6  /* combine with 1/K instead of routing weights */
};

double orc_e2m1(uint32_t nibble);
double orc_e4m3(uint32_t byte);       /* NaN for 0x7F / 0xFF */
double orc_bf16(uint16_t bits);
uint16_t orc_bf16_rne(double v);      /* nearest BF16, ties to even */
void orc_bf16_rne_array(int64_t n, const double *v, uint16_t *out);

/* Top-K of FP32 logits (NaN ranks below everything, ties -> lower id), ordered
 * descending; w[t][j] = exp(l_j - l_max) / sum over the K selected. Returns the
 * number of tokens whose selected logits are not all finite. */
int orc_route(int32_t T, int32_t E, int32_t K, const float *logits, int32_t *ids, double *w);

/* Number of tokens with an id outside [0,E) or a repeated id. */
int orc_check_ids(int32_t T, int32_t E, int32_t K, const int32_t *ids);

/* counts[E], offsets[E+1] (exclusive scan), perm[T*K] = pair index t*K+j grouped
 * by expert ascending, then by token ascending. ids must pass orc_check_ids. */
void orc_sort(int32_t T, int32_t E, int32_t K, const int32_t *ids, int32_t *counts,
              int32_t *offsets, int32_t *perm);

/* The quantiser that defines the synthetic weights: n_mat matrices [rows][cols]
 * of BF16 bits -> codes [n][rows][cols/2], scales [n][rows][cols/16], glob [n]. */
int orc_quantize(int32_t n_mat, int32_t rows, int32_t cols, const uint16_t *w_bf16,
                 uint8_t *codes, uint8_t *scales, float *glob);

/* Dense FP64 decode of one matrix of one expert: dst[rows][cols]. */
void orc_decode_matrix(int32_t rows, int32_t cols, const uint8_t *codes, const uint8_t *scales,
                       float glob, double *dst);

/* Router projection: logits[t][e] = sum_k bf16(w_r[e][k]) * x[t][k] in FP64, x FP32
 * [T][H] (never rounded to BF16), w_r BF16 bits [E][H]. */
void orc_router(int32_t T, int32_t E, int32_t H, const float *x, const uint16_t *w_r,
                double *logits);

/* The layer. act_type 0: act = BF16 bits [T][H]; 1: act = int8 [T][H] with
 * act_scale [T] (x = q * scale, the scale applied after the dot products).
 * ids [T][K], wts [T][K] (FP64). out [n][H] FP64 for the n tokens listed in
 * sample (sample == NULL: all T tokens, n = T). Tokens are split over nthreads
 * POSIX threads (<= 0: one per online core). Returns 0, or -1 on bad arguments. */
int orc_moe(const orc_dims *d, const orc_weights *w, int32_t T, int32_t act_type,
            const void *act, const float *act_scale, const int32_t *ids, const double *wts,
            int32_t n_sample, const int32_t *sample, double *out, int32_t nthreads,
            int32_t plant);

/* h (the SwiGLU output, FP64) of one (token, expert) pair: h[I]. */
int orc_pair_h(const orc_dims *d, const orc_weights *w, int32_t act_type, const void *x_row,
               float x_scale, int32_t e, double *h, int32_t plant);

#ifdef __cplusplus
}
#endif
#endif
