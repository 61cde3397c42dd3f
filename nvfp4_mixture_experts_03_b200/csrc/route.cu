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
#include "route_common.cuh"

namespace nvmoe {

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

// Kernel 2: one warp per expert: exclusive scan of its per-chunk counts (all
// loads issued first) -> cbase[e][c], and the expert's total -> counts[e].
__global__ void __launch_bounds__(1024) route_chunkscan_kernel(Params p) {
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (e >= p.E) return;
    const int *__restrict__ hrow = p.hist + (size_t)e * p.nch;
    int *__restrict__ crow = p.cbase + (size_t)e * p.nch;
    constexpr int kMaxIt = 32;   // nch <= 1024 chunks (T <= 65536)
    int v[kMaxIt];
#pragma unroll
    for (int i = 0; i < kMaxIt; i++) {
        const int c = 32 * i + lane;
        v[i] = c < p.nch ? hrow[c] : 0;
    }
    int carry = 0;
#pragma unroll
    for (int i = 0; i < kMaxIt; i++) {
        if (32 * i >= p.nch) break;
        int incl = v[i];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        const int c = 32 * i + lane;
        if (c < p.nch) crow[c] = carry + incl - v[i];
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) p.counts[e] = carry;
}

// Kernel 3 (one CTA of 1024 threads): expert offsets, the grouped-GEMM tile
// lists (experts with more than small_tok pairs) and the list of small experts.
__global__ void __launch_bounds__(1024) route_scan_kernel(Params p) {
    extern __shared__ int sm[];
    int *cnt_s = sm;                      // [E]
    int *off_s = cnt_s + p.E;             // [E+1]
    int *gub = off_s + p.E + 1;           // [E]
    int *dnb = gub + p.E;                 // [E]
    int *sml = dnb + p.E;                 // [E]
    int *wt = sml + p.E;                  // [33]
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) cnt_s[e] = p.counts[e];
    __syncthreads();
    const int mgu = cdiv(p.I, kGuRows), mdn = cdiv(p.H, kDnRows);
    auto small = [&](int c) { return c > 0 && c <= p.small_tok; };
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const int c = cnt_s[e];
        const int nt = small(c) ? 0 : cdiv(c, kBN);
        off_s[e] = c;
        gub[e] = nt * mgu;
        dnb[e] = nt * mdn;
        sml[e] = small(c) ? 1 : 0;
    }
    __syncthreads();
    const int total = block_exscan(off_s, p.E, wt);
    const int ngu = block_exscan(gub, p.E, wt);
    const int ndn = block_exscan(dnb, p.E, wt);
    const int nsm = block_exscan(sml, p.E, wt);
    if (threadIdx.x == 0) {
        off_s[p.E] = total;
        p.cnt[kCntTilesGu] = ngu;
        p.cnt[kCntTilesDn] = ndn;
        p.cnt[kCntSmall] = nsm;
        p.cnt[kCntSmallQ] = 0;
        p.cnt[kCntSmallQ + 1] = 0;
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
        p.offsets[e] = off_s[e];
        if (p.dbg_offsets) p.dbg_offsets[e] = off_s[e];
        if (e < p.E && p.dbg_counts) p.dbg_counts[e] = cnt_s[e];
        if (e < p.E && small(cnt_s[e])) p.small_e[sml[e]] = e;
    }
    for (int slot = threadIdx.x; slot < ngu; slot += blockDim.x)
        emit_tile(p.tiles_gu, gub, cnt_s, off_s, p.E, mgu, kGuRows, slot);
    for (int slot = threadIdx.x; slot < ndn; slot += blockDim.x)
        emit_tile(p.tiles_dn, dnb, cnt_s, off_s, p.E, mdn, kDnRows, slot);
}

// Kernel 4: positions of every pair of a 64-token chunk.
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


// One CTA per token: F16 copy of x_t scaled by 2^k (BF16/FP32 input) or the int8
// codes as F16 (exact), written to the position of each of the token's K pairs
// (the gate/up GEMM then loads contiguous 64-row boxes); and the scale that
// undoes it, per token and per pair position.
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
    const bool int8 = p.act_type == NVFP4_MOE_ACT_INT8;
    const int sh = int8 ? 0 : pow2_shift_for(amax);
    const float xs = int8 ? p.act_scale[t] : exp2i(-sh);
    // h of this token's pairs is stored times 2^he (the combine divides it out)
    const int he = h_exp_for(int8 ? 127.0f * xs : amax);
    if (threadIdx.x == 0) {
        p.xscale[t] = xs;
        p.phinv[t] = exp2i(-he);
    }
    if (threadIdx.x < p.K) {
        p.ps[spos[threadIdx.x]] = xs;
        p.ph[spos[threadIdx.x]] = exp2i(he);
    }
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
}

// -------------------------------------------------------------- combine

// out_t (+)= sum_j yp[pos(t, j)] over the token's K pairs, in the fixed order
// j = 0..K-1 with FP32 accumulation (yp holds w * s_d * y per pair, F16, in the
// buffer that held the pair-ordered activations). Resident CTAs stride over the
// tokens (one launch wave, no per-token CTA start-up); each thread issues all K
// loads of its 8 columns before adding them up.
__global__ void __launch_bounds__(256) combine_kernel(Params p) {
  for (int t = blockIdx.x; t < p.T; t += gridDim.x) {
    int spos[NVFP4_MOE_MAX_TOPK];
#pragma unroll
    for (int j = 0; j < NVFP4_MOE_MAX_TOPK; j++)
        if (j < p.K) spos[j] = __ldg(p.inv + (size_t)t * p.K + j);
    for (int k8 = threadIdx.x; k8 < p.H / 8; k8 += blockDim.x) {
        uint4 y[NVFP4_MOE_MAX_TOPK];
#pragma unroll
        for (int j = 0; j < NVFP4_MOE_MAX_TOPK; j++)
            if (j < p.K) y[j] = reinterpret_cast<const uint4 *>(p.xh + (size_t)spos[j] * p.H)[k8];
        float acc[8];
        float4 *o = reinterpret_cast<float4 *>(p.out + (size_t)t * p.H) + 2 * k8;
        if (p.out_add) {
            const float4 a = o[0], b = o[1];
            acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
            acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) acc[i] = 0.0f;
        }
        float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < NVFP4_MOE_MAX_TOPK; j++) {
            if (j < p.K) {
                const __half2 *hv = reinterpret_cast<const __half2 *>(&y[j]);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const float2 f = __half22float2(hv[i]);
                    sum[2 * i] += f.x;
                    sum[2 * i + 1] += f.y;
                }
            }
        }
        // the rows were built from h stored times 2^he of this token
        const float hinv = p.phinv[t];
        bool fin = true;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            acc[i] += sum[i] * hinv;
            fin &= isfinite(acc[i]);
        }
        if (!fin) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfOut | t);
        o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
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
    route_chunkscan_kernel<<<cdiv(p.E, 32), 1024, 0, s>>>(p);
    const size_t scan_bytes = (5 * p.E + 1 + 33) * sizeof(int);
    route_scan_kernel<<<1, 1024, scan_bytes, s>>>(p);
    route_scatter_kernel<<<p.nch, 256, mask_bytes, s>>>(p);
}

void launch_prep_prefill(const Params &p, cudaStream_t s) {
    prep_prefill_kernel<<<p.T, 256, 0, s>>>(p);
}

int sm_count();   // SMs of the current device (decode.cu)

void launch_combine(const Params &p, cudaStream_t s) {
    // eight 256-thread CTAs per SM (the SM's 2048 threads), fewer for short batches
    const int resident = 8 * sm_count();
    combine_kernel<<<p.T < resident ? p.T : resident, 256, 0, s>>>(p);
}


}  // namespace nvmoe
