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

// Orderable selection key: larger logit first, NaN below every number, equal
// logits -> lower expert id first. Key 0 marks an already chosen expert.
__device__ inline unsigned long long sel_key(float v, int e) {
    uint32_t o;
    if (isnan(v)) {
        o = 0;
    } else {
        uint32_t u = (v == 0.0f) ? 0u : __float_as_uint(v);
        o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    return ((unsigned long long)o << 32) | (uint32_t)(~(uint32_t)e);
}

// One warp selects the top-K of one token's logits (E <= 32*NPER). Lane j < K
// receives the j-th id and its renormalised weight.
template <int NPER>
__device__ inline void warp_topk(const float *__restrict__ row, int E, int K, int lane,
                                 int &my_id, float &my_w, bool &finite) {
    unsigned long long key[NPER];
#pragma unroll
    for (int i = 0; i < NPER; i++) {
        const int e = lane + 32 * i;
        key[i] = (e < E) ? sel_key(__ldg(row + e), e) : 0ull;
    }
    my_id = 0;
    float my_v = 0.0f;
    for (int j = 0; j < K; j++) {
        unsigned long long best = 0;
#pragma unroll
        for (int i = 0; i < NPER; i++) best = key[i] > best ? key[i] : best;
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            unsigned long long o = __shfl_xor_sync(0xffffffffu, best, off);
            best = o > best ? o : best;
        }
        const int e = (int)(~(uint32_t)(best & 0xffffffffull));
        if ((e & 31) == lane) {
#pragma unroll
            for (int i = 0; i < NPER; i++)
                if (i == (e >> 5)) key[i] = 0ull;
        }
        if (lane == j) {
            my_id = e;
            my_v = __ldg(row + e);
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

// Kernel 1: top-k for 64 tokens per CTA, then the chunk's per-expert counts.
template <int NPER>
__global__ void __launch_bounds__(256) route_topk_hist_kernel(Params p) {
    extern __shared__ uint32_t mask[];  // [2][E]
    const int c = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 2 * p.E; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    for (int i = 0; i < kChunkTokens / 8; i++) {
        const int tl = warp * (kChunkTokens / 8) + i;
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

// Writes the gate/up and down tile lists of the experts in [e_begin, e_end).
__device__ void emit_tiles(const Params &p, const int *cnt_s, const int *off_s, const int *gub,
                           const int *dnb, int e) {
    const int c = cnt_s[e];
    if (c == 0) return;
    const int nn = cdiv(c, kBN), mgu = p.I / kGuRows, mdn = p.H / kDnRows;
    for (int nt = 0; nt < nn; nt++) {
        const int pos0 = off_s[e] + nt * kBN, nk = min(kBN, c - nt * kBN);
        for (int mi = 0; mi < mgu; mi++)
            p.tiles_gu[gub[e] + nt * mgu + mi] = Tile{e, mi * kGuRows, pos0, nk};
        for (int mi = 0; mi < mdn; mi++)
            p.tiles_dn[dnb[e] + nt * mdn + mi] = Tile{e, mi * kDnRows, pos0, nk};
    }
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
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) emit_tiles(p, cnt_s, off_s, gub, dnb, e);
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

__device__ inline float load_act(const Params &p, int t, int k) {
    if (p.act_type == NVFP4_MOE_ACT_BF16)
        return __bfloat162float(((const __nv_bfloat16 *)p.act)[(size_t)t * p.H + k]);
    if (p.act_type == NVFP4_MOE_ACT_INT8) return (float)((const int8_t *)p.act)[(size_t)t * p.H + k];
    // FP32 residual stream: the layer's input is its BF16 rounding
    return __bfloat162float(__float2bfloat16_rn(((const float *)p.act)[(size_t)t * p.H + k]));
}

// One CTA per token: F16 copy of x_t scaled by 2^k (BF16/FP32 input) or the int8
// codes as F16 (exact), written to the position of each of the token's K pairs;
// the per-position scale that undoes it; and out_t cleared unless accumulating.
__global__ void __launch_bounds__(256) prep_prefill_kernel(Params p) {
    const int t = blockIdx.x;
    __shared__ float red[8];
    __shared__ int spos[NVFP4_MOE_MAX_TOPK];
    float amax = 0.0f;
    if (p.act_type != NVFP4_MOE_ACT_INT8)
        for (int k = threadIdx.x; k < p.H; k += blockDim.x) amax = fmaxf(amax, fabsf(load_act(p, t, k)));
#pragma unroll
    for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    if (threadIdx.x < p.K) spos[threadIdx.x] = p.inv[(size_t)t * p.K + threadIdx.x];
    __syncthreads();
    amax = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) amax = fmaxf(amax, red[w]);
    const int sh = (p.act_type == NVFP4_MOE_ACT_INT8) ? 0 : pow2_shift_for(amax);
    const float xs = (p.act_type == NVFP4_MOE_ACT_INT8) ? p.act_scale[t] : ldexpf(1.0f, -sh);
    if (threadIdx.x == 0) p.xscale[t] = xs;
    if (threadIdx.x < p.K) p.ps[spos[threadIdx.x]] = xs;
    // 8 elements per thread step -> one 16-byte store per pair
    for (int k8 = threadIdx.x; k8 < p.H / 8; k8 += blockDim.x) {
        __align__(16) __half v[8];
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = __float2half_rn(ldexpf(load_act(p, t, k8 * 8 + i), sh));
        const uint4 pk = *reinterpret_cast<const uint4 *>(v);
        for (int j = 0; j < p.K; j++)
            reinterpret_cast<uint4 *>(p.xh + (size_t)spos[j] * p.H)[k8] = pk;
    }
    if (!p.out_add)
        for (int k = threadIdx.x; k < p.H; k += blockDim.x) p.out[(size_t)t * p.H + k] = 0.0f;
}

// ---------------------------------------------------------------- small T

// One CTA, T <= 8: routing, counts, offsets, permutation, the unique-expert list
// with each (unique expert, token) position, the F16 activations and the
// output clear, in one launch.
template <int NPER>
__global__ void __launch_bounds__(256) route_small_kernel(Params p) {
    extern __shared__ int sm[];
    int *emask = sm;                  // [E] token bitmask per expert
    int *cnt_s = emask + p.E;         // [E] counts -> offsets
    int *flag = cnt_s + p.E;          // [E] 1 if used -> unique index
    int *wt = flag + p.E;             // [33]
    __shared__ int sid[NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK];
    __shared__ float sw[NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK];
    __shared__ float samax[NVFP4_MOE_DECODE_MAX_T];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) emask[e] = 0;
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
        // activation amax of this token (for the F16 shift)
        float amax = 0.0f;
        if (p.act_type != NVFP4_MOE_ACT_INT8)
            for (int k = lane; k < p.H; k += 32) amax = fmaxf(amax, fabsf(load_act(p, t, k)));
#pragma unroll
        for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) samax[t] = amax;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        cnt_s[e] = __popc(emask[e]);
        flag[e] = emask[e] != 0;
        p.counts[e] = cnt_s[e];
        if (p.dbg_counts) p.dbg_counts[e] = cnt_s[e];
    }
    __syncthreads();
    const int total = block_exscan(cnt_s, p.E, wt);
    const int U = block_exscan(flag, p.E, wt);
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
    for (int t = 0; t < p.T; t++) {
        const int sh = (p.act_type == NVFP4_MOE_ACT_INT8) ? 0 : pow2_shift_for(samax[t]);
        if (threadIdx.x == 0)
            p.xscale[t] = (p.act_type == NVFP4_MOE_ACT_INT8) ? p.act_scale[t] : ldexpf(1.0f, -sh);
        for (int k = threadIdx.x; k < p.H; k += blockDim.x)
            p.xh[(size_t)t * p.H + k] = __float2half_rn(ldexpf(load_act(p, t, k), sh));
        if (!p.out_add)
            for (int k = threadIdx.x; k < p.H; k += blockDim.x) p.out[(size_t)t * p.H + k] = 0.0f;
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
    NPER_SWITCH(p.E, (route_topk_hist_kernel<NP><<<p.nch, 256, mask_bytes, s>>>(p)));
    const size_t scan_bytes = (4 * p.E + 1 + 33) * sizeof(int);
    route_scan_kernel<<<1, 1024, scan_bytes, s>>>(p);
    route_scatter_kernel<<<p.nch, 256, mask_bytes, s>>>(p);
}

void launch_prep_prefill(const Params &p, cudaStream_t s) {
    prep_prefill_kernel<<<p.T, 256, 0, s>>>(p);
}

void launch_route_small(const Params &p, cudaStream_t s) {
    const size_t bytes = (3 * p.E + 33) * sizeof(int);
    NPER_SWITCH(p.E, (route_small_kernel<NP><<<1, 256, bytes, s>>>(p)));
}

}  // namespace nvmoe
