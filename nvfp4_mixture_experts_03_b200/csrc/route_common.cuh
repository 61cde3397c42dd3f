// Routing building blocks shared by the routing kernels and the decode kernels
// (which route their <= 8 tokens redundantly in every CTA): warp top-k with
// renormalised softmax weights, validation of precomputed routing, and a
// block-wide exclusive scan.
#pragma once
#include "common.cuh"

namespace nvmoe {

// Orderable 32-bit selection key: larger logit -> larger key; NaN -> 1 (below
// every number); 0 marks an expert already chosen. +0 and -0 share one key.
__device__ inline uint32_t sel_key(float v) {
    if (isnan(v)) return 1u;
    const uint32_t u = (v == 0.0f) ? 0u : __float_as_uint(v);
    const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return k < 2u ? 2u : k;  // -inf maps to 0x007FFFFF, so this never changes a number's order
}

// The logit a key came from (exact for every non-NaN key; +0 for the merged
// zeros; a NaN for the NaN key).
__device__ inline float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One warp selects the top-K of one token's logits (E <= 32*NPER): K rounds of
// (per-lane argmax over its NPER keys, warp max of the key, warp min of the
// expert id among lanes holding it), so equal logits go to the lower id. Lane
// j < K receives the j-th id and its renormalised weight.
template <int NPER>
__device__ inline void warp_topk(const float *__restrict__ row, int E, int K, int lane,
                                 int &my_id, float &my_w, bool &finite) {
    uint32_t key[NPER];
    // all loads first (clamped in-bounds addresses), so they are in flight together
#pragma unroll
    for (int i = 0; i < NPER; i++) key[i] = __float_as_uint(__ldg(row + min(lane + 32 * i, E - 1)));
#pragma unroll
    for (int i = 0; i < NPER; i++) key[i] = (lane + 32 * i < E) ? sel_key(__uint_as_float(key[i])) : 0u;
    my_id = 0;
    float my_v = 0.0f;
    for (int j = 0; j < K; j++) {
        uint32_t best = key[0];
        int bi = 0;
#pragma unroll
        for (int i = 1; i < NPER; i++)
            if (key[i] > best) { best = key[i]; bi = i; }   // strict: lowest i (lowest id) on ties
        const uint32_t gmax = __reduce_max_sync(0xffffffffu, best);
        const uint32_t cand = (best == gmax) ? (uint32_t)(lane + 32 * bi) : 0xffffffffu;
        const int e = (int)__reduce_min_sync(0xffffffffu, cand);
        const int hit = ((e & 31) == lane) ? (e >> 5) : -1;
#pragma unroll
        for (int i = 0; i < NPER; i++) key[i] = (i == hit) ? 0u : key[i];
        const float v = key_value(gmax);   // the selected logit, known to every lane
        if (lane == j) {
            my_id = e;
            my_v = v;
        }
    }
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = (lane < K) ? expf(my_v - vmax) : 0.0f;
    float den = 0.0f;
    for (int j = 0; j < K; j++) den += __shfl_sync(0xffffffffu, ex, j);  // fixed order j = 0..K-1
    my_w = ex / den;
    const bool fin = (lane >= K) || isfinite(my_v);
    finite = __all_sync(0xffffffffu, fin);
}

// Precomputed routing: lane j < K reads id/weight j. A token with an id out of
// range or a repeated id is reported (BAD_ROUTING) and neutralised: ids 0..K-1,
// weights 0, so every later index stays in bounds.
__device__ inline bool warp_given(const int32_t *ids, const float *w, int E, int K, int lane,
                                  int &my_id, float &my_w) {
    int id = (lane < K) ? ids[lane] : -1;
    float wv = (lane < K) ? w[lane] : 0.0f;
    bool ok = (lane >= K) || (id >= 0 && id < E);
    for (int j = 0; j < K; j++) {
        const int other = __shfl_sync(0xffffffffu, id, j);
        if (lane < K && j < lane && other == id) ok = false;
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (!all_ok) {
        id = lane;
        wv = 0.0f;
    }
    my_id = id;
    my_w = wv;
    return all_ok;
}

template <int NPER>
__device__ inline void route_token(const Params &p, int t, int lane, int &id, float &w) {
    if (p.logits) {
        bool finite;
        warp_topk<NPER>(p.logits + (size_t)t * p.E, p.E, p.K, lane, id, w, finite);
        if (!finite && lane == 0) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, t);
    } else {
        const bool ok = warp_given(p.in_ids + (size_t)t * p.K, p.in_w + (size_t)t * p.K, p.E, p.K,
                                   lane, id, w);
        if (!ok && lane == 0) latch_status(p.status, NVFP4_MOE_ERR_BAD_ROUTING, t);
    }
}

// In-place exclusive scan of n <= 32*blockDim ints in shared memory; returns the
// total. All threads of the block must call it.
__device__ inline int block_exscan(int *a, int n, int *warp_tot /* >= 32 */) {
    const int nt = blockDim.x, tid = threadIdx.x;
    const int per = (n + nt - 1) / nt;
    const int b = tid * per;
    int local = 0;
    for (int i = 0; i < per; i++)
        if (b + i < n) local += a[b + i];
    // warp inclusive scan of local
    const int lane = tid & 31, warp = tid >> 5;
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = nt >> 5;
        int v = lane < nw ? warp_tot[lane] : 0;
        int vi = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, vi, off);
            if (lane >= off) vi += o;
        }
        if (lane < nw) warp_tot[lane] = vi - v;  // exclusive warp offsets
        if (lane == nw - 1) warp_tot[32] = vi;   // grand total
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
    for (int i = 0; i < per; i++)
        if (b + i < n) {
            const int v = a[b + i];
            a[b + i] = run;
            run += v;
        }
    const int total = warp_tot[32];
    __syncthreads();
    return total;
}

// Eight consecutive activations (k8-th group of 8) of token t as FP32, with a
// 16-byte load (BF16, 8-byte for int8, two 16-byte loads for FP32).
__device__ inline void load_act8(const Params &p, int t, int k8, float (&v)[8]) {
    const size_t off = (size_t)t * p.H + 8 * k8;
    if (p.act_type == NVFP4_MOE_ACT_BF16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)p.act + off));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else if (p.act_type == NVFP4_MOE_ACT_INT8) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>((const int8_t *)p.act + off));
        const uint32_t w[2] = {u.x, u.y};
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = (float)(int8_t)(w[i >> 2] >> (8 * (i & 3)));
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>((const float *)p.act + off));
        const float4 b = __ldg(reinterpret_cast<const float4 *>((const float *)p.act + off) + 1);
        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = __bfloat162float(__float2bfloat16_rn(f[i]));
    }
}

// 2^sh as an FP32 (|sh| <= 120, so the exponent field stays normal).
__device__ inline float exp2i(int sh) { return __int_as_float((127 + sh) << 23); }

__device__ inline uint4 pack8_f16(const float (&v)[8], int sh) {
    const float m = exp2i(sh);  // exact power-of-two scaling
    __align__(16) __half hv[8];
#pragma unroll
    for (int i = 0; i < 8; i++) hv[i] = __float2half_rn(v[i] * m);
    return *reinterpret_cast<const uint4 *>(hv);
}

}  // namespace nvmoe
