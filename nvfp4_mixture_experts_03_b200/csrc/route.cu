// Routing: softmax top-k renormalised, per-expert histogram, exclusive scan,
// and the expert-grouped permutation of (token, slot) pairs.
//
// The pages ("Strata NVFP4" README, "How it differs from upstream Strata", the
// prompt-reading bullet) gather each expert group's work into one launch after
// one wait; here every count, offset and tile list is built on the device, so
// the grouped GEMMs that follow read their schedule without a host round trip.
//
// Order of the permutation: pairs grouped by expert ascending, then by token
// ascending (each token names an expert at most once). Ranks inside a chunk of
// 64 tokens come from per-expert 32-bit token masks, so the result is
// deterministic and needs no sort.
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

// One warp selects the top-K of one token's logits (E <= 32*NPER): K rounds of
// (per-lane argmax over its NPER keys, warp max of the key, warp min of the
// expert id among lanes holding it), so equal logits go to the lower id. Lane
// j < K receives the j-th id and its renormalised weight.
template <int NPER>
__device__ inline void warp_topk(const float *__restrict__ row, int E, int K, int lane,
                                 int &my_id, float &my_w, bool &finite) {
    uint32_t key[NPER];
    float val[NPER];
    // all loads first (clamped in-bounds addresses), so they are in flight together
#pragma unroll
    for (int i = 0; i < NPER; i++) val[i] = __ldg(row + min(lane + 32 * i, E - 1));
#pragma unroll
    for (int i = 0; i < NPER; i++) key[i] = (lane + 32 * i < E) ? sel_key(val[i]) : 0u;
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
        float v = 0.0f;
#pragma unroll
        for (int i = 0; i < NPER; i++) {
            v = (i == hit) ? val[i] : v;
            key[i] = (i == hit) ? 0u : key[i];
        }
        v = __shfl_sync(0xffffffffu, v, e & 31);
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

// ---------------------------------------------------------------- large T

// Kernel 1: top-k for 64 tokens per CTA (32 warps, 2 tokens each), then the
// chunk's per-expert counts.
template <int NPER>
constexpr int topk_threads() { return NPER >= 32 ? 512 : 1024; }

template <int NPER>
__global__ void __launch_bounds__(topk_threads<NPER>()) route_topk_hist_kernel(Params p) {
    extern __shared__ uint32_t mask[];  // [2][E]
    const int c = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 2 * p.E; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    const int per_warp = kChunkTokens / (int)(blockDim.x >> 5);
    for (int i = 0; i < per_warp; i++) {
        const int tl = warp * per_warp + i;
        const int t = c * kChunkTokens + tl;
        if (t >= p.T) break;
        int id;
        float w;
        route_token<NPER>(p, t, lane, id, w);
        if (lane < p.K) {
            p.ids[(size_t)t * p.K + lane] = id;
            p.wts[(size_t)t * p.K + lane] = w;
            if (p.dbg_ids) p.dbg_ids[(size_t)t * p.K + lane] = id;
            if (p.dbg_w) p.dbg_w[(size_t)t * p.K + lane] = w;
            atomicOr(&mask[(tl >> 5) * p.E + id], 1u << (tl & 31));
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        p.hist[(size_t)e * p.nch + c] = __popc(mask[e]) + __popc(mask[p.E + e]);
}

// In-place exclusive scan of n <= 32*blockDim ints in shared memory; returns the
// total. All threads of the block must call it.
__device__ int block_exscan(int *a, int n, int *warp_tot /* >= 32 */) {
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

// Tile slot -> (expert, n-tile, m-tile) by binary search over the per-expert
// exclusive tile offsets `base` (E entries, non-decreasing) in shared memory.
__device__ inline void emit_tile(Tile *tiles, const int *base, const int *cnt_s, const int *off_s,
                                 int E, int mt, int m_rows, int slot) {
    int lo = 0, hi = E - 1;  // last e with base[e] <= slot
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (base[mid] <= slot) lo = mid; else hi = mid - 1;
    }
    const int e = lo, r = slot - base[e];
    const int nt = r / mt, mi = r - nt * mt;
    const int pos0 = off_s[e] + nt * kBN;
    tiles[slot] = Tile{e, mi * m_rows, pos0, min(kBN, cnt_s[e] - nt * kBN)};
}

// Kernel 2 (one CTA of 1024 threads): per-expert scan over chunks, expert
// offsets, and the grouped-GEMM tile lists.
__global__ void __launch_bounds__(1024) route_scan_kernel(Params p) {
    extern __shared__ int sm[];
    int *cnt_s = sm;                      // [E]
    int *off_s = cnt_s + p.E;             // [E+1]
    int *gub = off_s + p.E + 1;           // [E]
    int *dnb = gub + p.E;                 // [E]
    int *wt = dnb + p.E;                  // [33]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int e = warp; e < p.E; e += nw) {
        int carry = 0;
        const int *hrow = p.hist + (size_t)e * p.nch;
        int *crow = p.cbase + (size_t)e * p.nch;
        for (int c0 = 0; c0 < p.nch; c0 += 32) {
            const int c = c0 + lane;
            const int v = c < p.nch ? hrow[c] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            if (c < p.nch) crow[c] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) cnt_s[e] = carry;
    }
    __syncthreads();
    const int mgu = p.I / kGuRows, mdn = p.H / kDnRows;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        off_s[e] = cnt_s[e];
        gub[e] = cdiv(cnt_s[e], kBN) * mgu;
        dnb[e] = cdiv(cnt_s[e], kBN) * mdn;
    }
    __syncthreads();
    const int total = block_exscan(off_s, p.E, wt);
    const int ngu = block_exscan(gub, p.E, wt);
    const int ndn = block_exscan(dnb, p.E, wt);
    if (threadIdx.x == 0) {
        off_s[p.E] = total;
        p.cnt[kCntTilesGu] = ngu;
        p.cnt[kCntTilesDn] = ndn;
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
        p.offsets[e] = off_s[e];
        if (p.dbg_offsets) p.dbg_offsets[e] = off_s[e];
        if (e < p.E) {
            p.counts[e] = cnt_s[e];
            if (p.dbg_counts) p.dbg_counts[e] = cnt_s[e];
        }
    }
    for (int slot = threadIdx.x; slot < ngu; slot += blockDim.x)
        emit_tile(p.tiles_gu, gub, cnt_s, off_s, p.E, mgu, kGuRows, slot);
    for (int slot = threadIdx.x; slot < ndn; slot += blockDim.x)
        emit_tile(p.tiles_dn, dnb, cnt_s, off_s, p.E, mdn, kDnRows, slot);
}

// Kernel 3: positions of every pair of a 64-token chunk.
__global__ void __launch_bounds__(256) route_scatter_kernel(Params p) {
    extern __shared__ uint32_t mask[];  // [2][E]
    const int c = blockIdx.x;
    for (int i = threadIdx.x; i < 2 * p.E; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    const int t0 = c * kChunkTokens;
    const int np = min(kChunkTokens, p.T - t0) * p.K;
    for (int q = threadIdx.x; q < np; q += blockDim.x) {
        const int tl = q / p.K;
        atomicOr(&mask[(tl >> 5) * p.E + p.ids[(size_t)t0 * p.K + q]], 1u << (tl & 31));
    }
    __syncthreads();
    for (int q = threadIdx.x; q < np; q += blockDim.x) {
        const int tl = q / p.K, pair = t0 * p.K + q;
        const int e = p.ids[pair];
        const uint32_t m = mask[(tl >> 5) * p.E + e] & ((1u << (tl & 31)) - 1u);
        const int rank = __popc(m) + ((tl >> 5) ? __popc(mask[e]) : 0);
        const int pos = p.offsets[e] + p.cbase[(size_t)e * p.nch + c] + rank;
        p.perm[pos] = pair;
        p.inv[pair] = pos;
        p.ptok[pos] = t0 + tl;
        p.pw[pos] = p.wts[pair];
        if (p.dbg_perm) p.dbg_perm[pos] = pair;
    }
}

// --------------------------------------------------------- activations prep


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

// One CTA per token: F16 copy of x_t scaled by 2^k (BF16/FP32 input) or the int8
// codes as F16 (exact), written to the position of each of the token's K pairs
// (the gate/up GEMM then loads contiguous 64-row boxes); the scale that undoes
// it, per token and per pair position; and out_t cleared unless accumulating.
__global__ void __launch_bounds__(256) prep_prefill_kernel(Params p) {
    const int t = blockIdx.x;
    __shared__ float red[8];
    __shared__ int spos[NVFP4_MOE_MAX_TOPK];
    constexpr int kMaxPer = 2;                  // 8-element groups per thread held in registers (H <= 4096)
    const int n8 = p.H / 8;
    float v[kMaxPer][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kMaxPer; i++) {
        const int k8 = threadIdx.x + i * blockDim.x;
        if (k8 < n8) {
            load_act8(p, t, k8, v[i]);
#pragma unroll
            for (int j = 0; j < 8; j++) amax = fmaxf(amax, fabsf(v[i][j]));
        }
    }
    for (int k8 = threadIdx.x + kMaxPer * blockDim.x; k8 < n8; k8 += blockDim.x) {  // H > 4096
        float w[8];
        load_act8(p, t, k8, w);
#pragma unroll
        for (int j = 0; j < 8; j++) amax = fmaxf(amax, fabsf(w[j]));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    if (threadIdx.x < p.K) spos[threadIdx.x] = p.inv[(size_t)t * p.K + threadIdx.x];
    __syncthreads();
    amax = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) amax = fmaxf(amax, red[w]);
    const int sh = (p.act_type == NVFP4_MOE_ACT_INT8) ? 0 : pow2_shift_for(amax);
    const float xs = (p.act_type == NVFP4_MOE_ACT_INT8) ? p.act_scale[t] : exp2i(-sh);
    if (threadIdx.x == 0) p.xscale[t] = xs;
    if (threadIdx.x < p.K) p.ps[spos[threadIdx.x]] = xs;
#pragma unroll
    for (int i = 0; i < kMaxPer; i++) {
        const int k8 = threadIdx.x + i * blockDim.x;
        if (k8 < n8) {
            const uint4 pk = pack8_f16(v[i], sh);
            for (int j = 0; j < p.K; j++) reinterpret_cast<uint4 *>(p.xh + (size_t)spos[j] * p.H)[k8] = pk;
        }
    }
    for (int k8 = threadIdx.x + kMaxPer * blockDim.x; k8 < n8; k8 += blockDim.x) {
        float w[8];
        load_act8(p, t, k8, w);
        const uint4 pk = pack8_f16(w, sh);
        for (int j = 0; j < p.K; j++) reinterpret_cast<uint4 *>(p.xh + (size_t)spos[j] * p.H)[k8] = pk;
    }
    if (!p.out_add)
        for (int k4 = threadIdx.x; k4 < p.H / 4; k4 += blockDim.x)
            reinterpret_cast<float4 *>(p.out + (size_t)t * p.H)[k4] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------- small T

// One CTA, T <= 8: routing, counts, offsets, permutation, the unique-expert list
// with each (unique expert, token) position, the F16 activations and the
// output clear, in one launch.
constexpr int kSmallThreads = 512;

template <int NPER>
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(Params p) {
    extern __shared__ int sm[];
    int *emask = sm;                  // [E] token bitmask per expert
    int *cnt_s = emask + p.E;         // [E] counts -> offsets
    int *flag = cnt_s + p.E;          // [E] 1 if used -> unique index
    int *wt = flag + p.E;             // [33]
    __shared__ int sid[NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK];
    __shared__ float sw[NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK];
    __shared__ unsigned samax_u[NVFP4_MOE_DECODE_MAX_T];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) emask[e] = 0;
    if (threadIdx.x < NVFP4_MOE_DECODE_MAX_T) samax_u[threadIdx.x] = 0u;
    __syncthreads();
    if (warp < p.T) {
        const int t = warp;
        int id;
        float w;
        route_token<NPER>(p, t, lane, id, w);
        if (lane < p.K) {
            sid[t * p.K + lane] = id;
            sw[t * p.K + lane] = w;
            p.ids[t * p.K + lane] = id;
            p.wts[t * p.K + lane] = w;
            if (p.dbg_ids) p.dbg_ids[t * p.K + lane] = id;
            if (p.dbg_w) p.dbg_w[t * p.K + lane] = w;
            atomicOr(&emask[id], 1 << t);
        }
    }
    // per-token activation amax (for the F16 shift): 16-byte loads from all threads
    if (p.act_type != NVFP4_MOE_ACT_INT8) {
        const int n8 = p.H / 8;
#pragma unroll 4
        for (int c = threadIdx.x; c < p.T * n8; c += blockDim.x) {
            float v[8];
            load_act8(p, c / n8, c % n8, v);
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; j++) m = fmaxf(m, fabsf(v[j]));
            atomicMax(&samax_u[c / n8], __float_as_uint(m));   // non-negative: integer order
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const int c = __popc(emask[e]);
        cnt_s[e] = c | ((c != 0) << 16);   // one scan: pairs (low 16 bits), used experts (high)
        p.counts[e] = c;
        if (p.dbg_counts) p.dbg_counts[e] = c;
    }
    __syncthreads();
    const int both = block_exscan(cnt_s, p.E, wt);
    const int total = both & 0xFFFF, U = both >> 16;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        flag[e] = cnt_s[e] >> 16;
        cnt_s[e] &= 0xFFFF;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        p.cnt[kCntUniq] = U;
        p.offsets[p.E] = total;
        if (p.dbg_offsets) p.dbg_offsets[p.E] = total;
    }
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        p.offsets[e] = cnt_s[e];
        if (p.dbg_offsets) p.dbg_offsets[e] = cnt_s[e];
        const int m = emask[e];
        if (m) {
            const int u = flag[e];
            p.uniq[u] = e;
            for (int t = 0; t < NVFP4_MOE_DECODE_MAX_T; t++)
                p.upos[u * NVFP4_MOE_DECODE_MAX_T + t] =
                    ((m >> t) & 1) ? cnt_s[e] + __popc(m & ((1 << t) - 1)) : -1;
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < p.T * p.K; q += blockDim.x) {
        const int t = q / p.K, e = sid[q];
        const int pos = cnt_s[e] + __popc(emask[e] & ((1 << t) - 1));
        p.perm[pos] = q;
        p.inv[q] = pos;
        p.ptok[pos] = t;
        p.pw[pos] = sw[q];
        if (p.dbg_perm) p.dbg_perm[pos] = q;
    }
    if (threadIdx.x < p.T) {
        const int t = threadIdx.x;
        const int sh = (p.act_type == NVFP4_MOE_ACT_INT8) ? 0 : pow2_shift_for(__uint_as_float(samax_u[t]));
        p.xscale[t] = (p.act_type == NVFP4_MOE_ACT_INT8) ? p.act_scale[t] : exp2i(-sh);
    }
    {
        const int n8 = p.H / 8;
#pragma unroll 4
        for (int c = threadIdx.x; c < p.T * n8; c += blockDim.x) {
            const int t = c / n8;
            const int sh = (p.act_type == NVFP4_MOE_ACT_INT8) ? 0 : pow2_shift_for(__uint_as_float(samax_u[t]));
            float v[8];
            load_act8(p, t, c % n8, v);
            reinterpret_cast<uint4 *>(p.xh)[c] = pack8_f16(v, sh);
        }
        if (!p.out_add)
            for (int c = threadIdx.x; c < p.T * p.H / 4; c += blockDim.x)
                reinterpret_cast<float4 *>(p.out)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ------------------------------------------------------------------ launch

#define NPER_SWITCH(E, ...)                                  \
    do {                                                     \
        const int _n = cdiv((E), 32);                        \
        if (_n <= 1) { constexpr int NP = 1; __VA_ARGS__; }       \
        else if (_n <= 2) { constexpr int NP = 2; __VA_ARGS__; }  \
        else if (_n <= 4) { constexpr int NP = 4; __VA_ARGS__; }  \
        else if (_n <= 8) { constexpr int NP = 8; __VA_ARGS__; }  \
        else if (_n <= 16) { constexpr int NP = 16; __VA_ARGS__; } \
        else { constexpr int NP = 32; __VA_ARGS__; }              \
    } while (0)

void launch_route_large(const Params &p, cudaStream_t s) {
    const size_t mask_bytes = 2 * p.E * sizeof(uint32_t);
    NPER_SWITCH(p.E, (route_topk_hist_kernel<NP><<<p.nch, topk_threads<NP>(), mask_bytes, s>>>(p)));
    const size_t scan_bytes = (4 * p.E + 1 + 33) * sizeof(int);
    route_scan_kernel<<<1, 1024, scan_bytes, s>>>(p);
    route_scatter_kernel<<<p.nch, 256, mask_bytes, s>>>(p);
}

void launch_prep_prefill(const Params &p, cudaStream_t s) {
    prep_prefill_kernel<<<p.T, 256, 0, s>>>(p);
}

void launch_route_small(const Params &p, cudaStream_t s) {
    const size_t bytes = (3 * p.E + 33) * sizeof(int);
    NPER_SWITCH(p.E, (route_small_kernel<NP><<<1, kSmallThreads, bytes, s>>>(p)));
}

}  // namespace nvmoe
