// Decode path (T <= 8): stream each selected expert's 4.5-bit weights once.
//
// The pages keep the quality profile on "canonical FP32 expert decode" ("#1858
// ... strata-safetensors", "What do you want to do?" and the paragraph after
// the measurements) and note that a decode round is bound by moving expert
// bytes ("Strata NVFP4" README, "Limits"). On B200 every expert is resident in
// HBM, so decode is a pure HBM stream whose time is set by how early the weight
// loads start, how many are in flight, and how evenly the bytes are spread.
//
// One kernel per layer, one 16-warp CTA per SM, launched with programmatic
// dependent launch (each CTA lets the next layer's grid launch once its own work
// is done):
//   routing: every CTA routes the <= 8 tokens itself (warp top-k per token, then
//     the <= 128 (token, slot) pairs ranked by (expert, token) to give positions,
//     the used-expert list and each (expert, token) position and weight);
//   phase 1 (gate/up + SwiGLU): the units (used expert, 8 intermediates, 128-wide
//     K round) are cut into equal contiguous ranges, one per warp of the grid.
//     A warp that covers a whole item applies SwiGLU to its registers; partial
//     items add their FP32 sums into a per-handle accumulator, and the warp whose
//     contribution completes the item applies SwiGLU from there (clearing it).
//     Every finished item counts towards its expert's ready count;
//   phase 2 (down + weighted combine): the units (used expert, 16 hidden rows,
//     128-wide K round) are cut into equal contiguous ranges, one per CTA (split
//     evenly over its warps). A CTA issues its first weight loads, waits only for
//     the ready counts of the one or two experts its range touches, copies their
//     h rows into shared memory, and adds its partial sums into out.
// No grid-wide barrier: the only cross-CTA waits are the per-expert ready counts
// and one count of CTAs that have read the activations (out may alias them),
// all bounded. The last CTA past its waits resets the counts, at its end, for
// the next launch.
// Arithmetic: each weight is decoded exactly to F16 (E2M1 -> F16 conversion
// times its E4M3 group scale: at most 6 significant bits, exact in F16) and fed
// to mma.sync m16n8k16 with the token slots as N, FP32 accumulation; the tensor
// scale and the per-token activation scale are applied to the FP32 result.
//
// Fragment mapping (m16n8k16, A row-major, B col-major): thread (g = lane/4,
// q = lane%4) holds rows g and g+8. It loads 16 contiguous code bytes of each
// row per 128-wide K round (byte offset 64*r + 16*q), so a warp reads whole
// 32-byte sectors. Mma step s of round r uses physical K 128r + 32q + 4s +
// {0,1,2,3} for logical K {2q, 2q+1, 2q+8, 2q+9}; the activations use the same
// permutation, so every dot product is the plain one.
#include "common.cuh"
#include "route_common.cuh"

namespace nvmoe {

__device__ inline uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ inline void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// Eight mma steps of one 128-wide K round: A rows (g: ca, g+8: cb) as 16 code
// bytes each with their two group scales; B from `bfrag(s)`.
template <class BF>
__device__ inline void round_mma(float (&acc)[4], const uint4 &ca, const uint4 &cb, uint32_t sa,
                                 uint32_t sb, BF bfrag) {
    const uint32_t sa0 = e4m3_to_f16x2_bcast(sa & 0xFF), sa1 = e4m3_to_f16x2_bcast(sa >> 8);
    const uint32_t sb0 = e4m3_to_f16x2_bcast(sb & 0xFF), sb1 = e4m3_to_f16x2_bcast(sb >> 8);
    const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w}, wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
    for (int w = 0; w < 4; w++) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        e2m1x8_to_f16(wa[w], a0, a1, a2, a3);   // bytes 4w..4w+3 of row g
        e2m1x8_to_f16(wb[w], b0, b1, b2, b3);   // same bytes of row g+8
        const uint32_t s_a = w < 2 ? sa0 : sa1, s_b = w < 2 ? sb0 : sb1;
        uint32_t x0, x1;
        bfrag(2 * w, x0, x1);
        mma_16816(acc, hmul2(a0, s_a), hmul2(b0, s_b), hmul2(a1, s_a), hmul2(b1, s_b), x0, x1);
        bfrag(2 * w + 1, x0, x1);
        mma_16816(acc, hmul2(a2, s_a), hmul2(b2, s_b), hmul2(a3, s_a), hmul2(b3, s_b), x0, x1);
    }
}


constexpr int kDecWarps = 16;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kMaxRoundsPerWarp = 4;   // 128-wide K rounds of loads one warp holds per chunk
constexpr int kMaxPairs = NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK;  // 128
constexpr int kSlots = NVFP4_MOE_DECODE_MAX_T;
constexpr uint64_t kDecWaitNs = 200000000ull;

// Per-CTA routing state of the decode kernel.
struct DecRoute {
    int ids[kMaxPairs];
    float w[kMaxPairs];
    int pos[kMaxPairs];             // position of pair q (grouped by expert, then token)
    int sorted_e[kMaxPairs];        // expert at each position
    int uniq[kMaxPairs];            // used experts, ascending
    int uoff[kMaxPairs + 1];        // first position of each used expert; uoff[U] = P
    int upos[kMaxPairs * kSlots];   // pair position of (used expert, token), -1 if absent
    float uw[kMaxPairs * kSlots];   // routing weight of (used expert, token)
    unsigned amax[kSlots];          // per-token activation amax (FP32 bits)
    float xsc[kSlots];              // per-token factor that undoes the F16 staging scale
    int U;
};

// Routes the T <= 8 tokens inside one CTA (identical result in every CTA).
template <int NPER>
__device__ void cta_route(const Params &p, DecRoute &R, bool report) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.T * p.K;
    for (int i = threadIdx.x; i < kMaxPairs * kSlots; i += blockDim.x) R.upos[i] = -1;
    if (warp < p.T) {
        int id;
        float w;
        if (p.logits) {
            bool finite;
            warp_topk<NPER>(p.logits + (size_t)warp * p.E, p.E, p.K, lane, id, w, finite);
            if (!finite && report && lane == 0) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, warp);
        } else {
            const bool ok = warp_given(p.in_ids + (size_t)warp * p.K, p.in_w + (size_t)warp * p.K,
                                       p.E, p.K, lane, id, w);
            if (!ok && report && lane == 0) latch_status(p.status, NVFP4_MOE_ERR_BAD_ROUTING, warp);
        }
        if (lane < p.K) {
            R.ids[warp * p.K + lane] = id;
            R.w[warp * p.K + lane] = w;
        }
    }
    __syncthreads();
    // A token's ids are distinct, so ordering the pairs q = t*K + j by (expert, q)
    // groups them by expert and, within an expert, by token.
    const int q = threadIdx.x;
    int e = 0, rank = 0;
    if (q < P) {
        e = R.ids[q];
        const int key = (e << 7) | q;
        for (int j = 0; j < P; j++) rank += ((R.ids[j] << 7) | j) < key;
        R.pos[q] = rank;
        R.sorted_e[rank] = e;
    }
    __syncthreads();
    const bool first = q < P && (rank == 0 || R.sorted_e[rank - 1] != e);
    const int U = __syncthreads_count(first);
    if (first) {
        int u = 0;   // distinct experts at positions before this one
        for (int j = 1; j < rank; j++) u += R.sorted_e[j] != R.sorted_e[j - 1];
        u += rank > 0;
        R.uniq[u] = e;
        R.uoff[u] = rank;
    }
    if (threadIdx.x == 0) {
        R.U = U;
        R.uoff[U] = P;
    }
    __syncthreads();
    if (q < P) {
        int lo = 0, hi = U - 1;   // u of this pair's expert (uniq ascending)
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (R.uniq[mid] <= e) lo = mid; else hi = mid - 1;
        }
        const int t = q / p.K;
        R.upos[lo * kSlots + t] = rank;
        R.uw[lo * kSlots + t] = R.w[q];
    }
    __syncthreads();
}

// The routing results a forward call leaves in the workspace (and the optional
// debug copies); written by CTA 0.
__device__ void publish_route(const Params &p, const DecRoute &R) {
    const int P = p.T * p.K;
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
        const int pos = R.pos[q], t = q / p.K;
        p.ids[q] = R.ids[q];
        p.wts[q] = R.w[q];
        p.perm[pos] = q;
        p.inv[q] = pos;
        p.ptok[pos] = t;
        p.pw[pos] = R.w[q];
        if (p.dbg_ids) p.dbg_ids[q] = R.ids[q];
        if (p.dbg_w) p.dbg_w[q] = R.w[q];
        if (p.dbg_perm) p.dbg_perm[pos] = q;
    }
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
        int before = 0, at = 0;
        for (int j = 0; j < P; j++) {
            before += R.ids[j] < e;
            at += R.ids[j] == e;
        }
        p.offsets[e] = before;
        if (p.dbg_offsets) p.dbg_offsets[e] = before;
        if (e < p.E) {
            p.counts[e] = at;
            if (p.dbg_counts) p.dbg_counts[e] = at;
        }
    }
    if (threadIdx.x == 0) p.cnt[kCntUniq] = R.U;
}

// One pass's weight data of one warp: rows g and g+8, up to kMaxRoundsPerWarp rounds.
struct PassBuf {
    uint4 ca[kMaxRoundsPerWarp], cb[kMaxRoundsPerWarp];
    uint32_t sa[kMaxRoundsPerWarp], sb[kMaxRoundsPerWarp];
};

struct ItemRef {
    int u, e, m0;
    bool valid;
};

// A run of at most kMaxRoundsPerWarp consecutive K rounds of one item.
struct Chunk {
    int item, r0, r1;   // r1 == 0: none
};

// Next chunk of the unit range [x, end) (units = item * R + round); advances x.
__device__ inline Chunk take_chunk(int &x, int end, int R) {
    Chunk c{0, 0, 0};
    if (x < end) {
        c.item = x / R;
        c.r0 = x - c.item * R;
        c.r1 = min(min(R, c.r0 + kMaxRoundsPerWarp), end - c.item * R);
        x = c.item * R + c.r1;
    }
    return c;
}

// MODE 0 item = (used expert u, 8 intermediates): A rows g are gate rows, rows
// g+8 the up rows of the same intermediate index. MODE 1 item = (u, 16 hidden
// rows).
template <int MODE>
__device__ inline ItemRef item_of(const Params &p, const DecRoute &R, const Chunk &c) {
    ItemRef r{0, 0, 0, c.r1 > 0};
    if (r.valid) {
        const int per_u = MODE == 0 ? p.I / 8 : p.H / 16;
        r.u = c.item / per_u;
        r.m0 = (c.item - r.u * per_u) * (MODE == 0 ? 8 : 16);
        r.e = R.uniq[r.u];
    }
    return r;
}

template <int MODE>
__device__ inline void issue_loads(const Params &p, const ItemRef &it, int g, int q, int r_begin,
                                   int r_end, PassBuf &b) {
    if (!it.valid) return;
    const int H = p.H, I = p.I;
    const uint8_t *ca_p, *cb_p, *sa_p, *sb_p;
    if (MODE == 0) {
        const size_t ra = (size_t)it.e * I + it.m0 + g;
        ca_p = p.gate_codes + ra * (H / 2);
        cb_p = p.up_codes + ra * (H / 2);
        sa_p = p.gate_scales + ra * (H / 16);
        sb_p = p.up_scales + ra * (H / 16);
    } else {
        const size_t ra = (size_t)it.e * H + it.m0 + g;
        ca_p = p.down_codes + ra * (I / 2);
        cb_p = p.down_codes + (ra + 8) * (I / 2);
        sa_p = p.down_scales + ra * (I / 16);
        sb_p = p.down_scales + (ra + 8) * (I / 16);
    }
#pragma unroll
    for (int j = 0; j < kMaxRoundsPerWarp; j++) {
        const int r = r_begin + j;
        if (r < r_end) {
            b.ca[j] = ldg_stream(ca_p + 64 * r + 16 * q);
            b.cb[j] = ldg_stream(cb_p + 64 * r + 16 * q);
            b.sa[j] = __ldg(reinterpret_cast<const unsigned short *>(sa_p + 8 * r + 2 * q));
            b.sb[j] = __ldg(reinterpret_cast<const unsigned short *>(sb_p + 8 * r + 2 * q));
        }
    }
}

__device__ inline void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}

// Raw activation bytes per token held in shared memory (0: FP32 input, which is
// read from global memory instead).
__host__ __device__ inline int raw_act_bytes(int act_type, int H) {
    return act_type == NVFP4_MOE_ACT_BF16 ? 2 * H : (act_type == NVFP4_MOE_ACT_INT8 ? H : 0);
}

// Eight activations of token t (group k8) as FP32, from the shared raw copy when
// there is one, else from global memory.
__device__ inline void act8(const Params &p, const uint8_t *raw, int t, int k8, float (&v)[8]) {
    if (p.act_type == NVFP4_MOE_ACT_BF16) {
        const uint4 u = reinterpret_cast<const uint4 *>(raw + (size_t)t * 2 * p.H)[k8];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else if (p.act_type == NVFP4_MOE_ACT_INT8) {
        const uint2 u = reinterpret_cast<const uint2 *>(raw + (size_t)t * p.H)[k8];
        const uint32_t w[2] = {u.x, u.y};
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = (float)(int8_t)(w[i >> 2] >> (8 * (i & 3)));
    } else {
        load_act8(p, t, k8, v);
    }
}


// Bounded wait until *word >= target (one thread); latches TIMEOUT on give-up.
__device__ inline bool wait_geq(const int32_t *word, int target, int32_t *status, int where) {
    const volatile int32_t *v = word;
    if (*v >= target) return true;
    const uint64_t t0 = globaltimer();
    while (*v < target) {
        __nanosleep(64);
        if (globaltimer() - t0 > kDecWaitNs) {
            latch_status(status, NVFP4_MOE_ERR_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

struct DecSmem {
    __half *xs;     // [8 token slots][H+4] F16 activations
    uint8_t *raw;   // [T][H] raw BF16 / int8 activations (cp.async at kernel start)
    __half *hs;     // [hs_rows][I+8] h rows of this CTA's phase-2 experts
};

// Phase 1 end of an item segment (nr rounds of the item's R1 done here).
__device__ inline void flush_gateup(const Params &p, const DecRoute &R, const ItemRef &it, int nr,
                                    int R1, const float (&acc)[4], int g, int q, int lane) {
    const int I = p.I;
    const int item = it.u * (I / 8) + it.m0 / 8;
    int32_t *ds = p.dstate;
    float *gu = p.dgu;
    bool finisher = true;
    if (nr != R1) {
#pragma unroll
        for (int c = 0; c < 2; c++) {
            const int tok = 2 * q + c;
            const int pos = tok < p.T ? R.upos[it.u * kSlots + tok] : -1;
            if (pos >= 0) {
                atomicAdd(gu + ((size_t)2 * pos) * I + it.m0 + g, acc[c]);
                atomicAdd(gu + ((size_t)2 * pos + 1) * I + it.m0 + g, acc[2 + c]);
            }
        }
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            __threadfence();
            last = atomicAdd(ds + kDsItems + item, nr) + nr == R1;
        }
        finisher = __shfl_sync(0xffffffffu, last, 0) != 0;
        if (!finisher) return;
        __threadfence();
    }
    const float sg = p.gate_global[it.e], su = p.up_global[it.e];
#pragma unroll
    for (int c = 0; c < 2; c++) {
        const int tok = 2 * q + c;
        const int pos = tok < p.T ? R.upos[it.u * kSlots + tok] : -1;
        if (pos >= 0) {
            float gs = acc[c], us = acc[2 + c];
            if (nr != R1) {   // the item's full sums; leaves the accumulator cleared
                gs = atomicExch(gu + ((size_t)2 * pos) * I + it.m0 + g, 0.0f);
                us = atomicExch(gu + ((size_t)2 * pos + 1) * I + it.m0 + g, 0.0f);
            }
            const float gv = gs * sg * R.xsc[tok], uv = us * su * R.xsc[tok];
            const float hf = silu(gv) * uv;
            if (!fits_f16(hf)) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfH | it.e);
            p.h[(size_t)pos * I + it.m0 + g] = __float2half_rn(hf);
        }
    }
    __syncwarp();
    if (lane == 0) {
        if (nr != R1) atomicExch(ds + kDsItems + item, 0);
        __threadfence();
        atomicAdd(ds + kDsReady + it.u, 1);
    }
}

// Phase 2 end of an item segment: the weighted partial sums into out.
__device__ inline void flush_down(const Params &p, const DecRoute &R, const ItemRef &it,
                                  const float (&acc)[4], int g, int q) {
    const float sd = p.down_global[it.e];
#pragma unroll
    for (int c = 0; c < 2; c++) {
        const int tok = 2 * q + c;
        if (tok < p.T && R.upos[it.u * kSlots + tok] >= 0) {
            const float w = R.uw[it.u * kSlots + tok] * sd;
            const float y0 = acc[c] * w, y1 = acc[2 + c] * w;
            if (!isfinite(y0) || !isfinite(y1)) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfY | it.e);
            atomicAdd(p.out + (size_t)tok * p.H + it.m0 + g, y0);
            atomicAdd(p.out + (size_t)tok * p.H + it.m0 + g + 8, y1);
        }
    }
}

// Streams the warp's unit range [x, end) of one projection; `cur` (already in
// buf0) is its first chunk. Loads of the next chunk are issued before the current
// chunk computes (two register buffers).
template <int MODE>
__device__ inline void run_range(const Params &p, const DecRoute &R, const DecSmem &S, int &x,
                                 int end, Chunk cur, PassBuf &buf0, PassBuf &buf1, int hs_pos0) {
    const int H = p.H, I = p.I, T = p.T;
    const int RR = (MODE == 0 ? H : I) / 128;
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int ld = H + 4, ldh = I + 8;
    const __half *xrow = S.xs + g * ld + 32 * q;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int seg_r0 = cur.r0;

    auto step = [&](PassBuf &b, PassBuf &nb) {
        const Chunk nxt = take_chunk(x, end, RR);
        issue_loads<MODE>(p, item_of<MODE>(p, R, nxt), g, q, nxt.r0, nxt.r1, nb);
        const ItemRef it = item_of<MODE>(p, R, cur);
        const int mypos = (MODE == 1 && g < T) ? R.upos[it.u * kSlots + g] : -1;
        const __half *hrow = S.hs + (size_t)(mypos < 0 ? 0 : mypos - hs_pos0) * ldh + 32 * q;
#pragma unroll
        for (int j = 0; j < kMaxRoundsPerWarp; j++) {
            const int r = cur.r0 + j;
            if (r < cur.r1) {
                if (MODE == 0) {
                    const __half *xr = xrow + 128 * r;
                    round_mma(acc, b.ca[j], b.cb[j], b.sa[j], b.sb[j],
                              [&](int s, uint32_t &x0, uint32_t &x1) {
                                  const uint2 v = *reinterpret_cast<const uint2 *>(xr + 4 * s);
                                  x0 = v.x;
                                  x1 = v.y;
                              });
                } else {
                    uint4 hv[4];
#pragma unroll
                    for (int v = 0; v < 4; v++)
                        hv[v] = mypos >= 0 ? reinterpret_cast<const uint4 *>(hrow + 128 * r)[v]
                                           : make_uint4(0, 0, 0, 0);
                    round_mma(acc, b.ca[j], b.cb[j], b.sa[j], b.sb[j],
                              [&](int s, uint32_t &x0, uint32_t &x1) {
                                  const uint4 &w = hv[s >> 1];
                                  x0 = (s & 1) ? w.z : w.x;
                                  x1 = (s & 1) ? w.w : w.y;
                              });
                }
            }
        }
        if (nxt.r1 == 0 || nxt.item != cur.item) {
            if (MODE == 0)
                flush_gateup(p, R, it, cur.r1 - seg_r0, RR, acc, g, q, lane);
            else
                flush_down(p, R, it, acc, g, q);
#pragma unroll
            for (int c = 0; c < 4; c++) acc[c] = 0.0f;
            seg_r0 = nxt.r0;
        }
        cur = nxt;
    };
    while (cur.r1 > 0) {
        step(buf0, buf1);
        if (cur.r1 == 0) break;
        step(buf1, buf0);
    }
}

// [a, b) = this warp's share of n units when the grid's W workers split them
// evenly in contiguous ranges.
__device__ inline void share(int n, int w, int W, int &a, int &b) {
    a = (int)((long long)n * w / W);
    b = (int)((long long)n * (w + 1) / W);
}

template <int NPER>
__global__ void __launch_bounds__(kDecThreads, 1) decode_layer_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ DecRoute R;
    const int H = p.H, I = p.I, T = p.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ld = H + 4;
    DecSmem S;
    S.xs = reinterpret_cast<__half *>(dsm);
    S.raw = reinterpret_cast<uint8_t *>(S.xs + kSlots * ld);
    S.hs = reinterpret_cast<__half *>(S.raw + T * raw_act_bytes(p.act_type, H));
    int32_t *ds = p.dstate;

    // Everything this layer reads may come from the previous kernel in the stream.
    grid_dep_wait();

    // the activations first: their loads are then not queued behind the weights'
    const int raw_bytes = T * raw_act_bytes(p.act_type, H);
    for (int c = threadIdx.x; c < raw_bytes / 16; c += blockDim.x)
        cp_async16(S.raw + 16 * c, static_cast<const uint8_t *>(p.act) + 16 * c);
    asm volatile("cp.async.commit_group;" ::: "memory");

    cta_route<NPER>(p, R, blockIdx.x == 0);
    const int U = R.U;

    // phase-1 share of this warp and its first loads
    const int R1 = H / 128, R2 = I / 128;
    const int n1 = U * (I / 8) * R1, n2 = U * (H / 16) * R2;
    int a1, b1;
    share(n1, blockIdx.x * kDecWarps + warp, gridDim.x * kDecWarps, a1, b1);
    int x1 = a1;
    const Chunk c1 = take_chunk(x1, b1, R1);
    PassBuf buf0, buf1;

    // per-token amax -> power-of-two shift -> F16 activations in shared memory
    // (token slots past T are zeros)
    const int n8 = H / 8;
    for (int c = threadIdx.x; c < (kSlots - T) * n8; c += blockDim.x) {
        uint2 *dst = reinterpret_cast<uint2 *>(S.xs + (T + c / n8) * ld + 8 * (c % n8));
        dst[0] = make_uint2(0, 0);
        dst[1] = make_uint2(0, 0);
    }
    if (threadIdx.x < kSlots) R.amax[threadIdx.x] = 0u;
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    const int ngrp = T * n8, ngrp_w = (ngrp + 31) & ~31;
    if (p.act_type != NVFP4_MOE_ACT_INT8) {
        for (int c = threadIdx.x; c < ngrp_w; c += blockDim.x) {
            float m = 0.0f;
            if (c < ngrp) {
                float v[8];
                act8(p, S.raw, c / n8, c % n8, v);
#pragma unroll
                for (int j = 0; j < 8; j++) m = fmaxf(m, fabsf(v[j]));
            }
            // a warp's 32 groups span at most two tokens (n8 is a multiple of 16)
            const unsigned t = (unsigned)min(c / n8, kSlots - 1);
            const unsigned lo_t = __shfl_sync(0xffffffffu, t, 0);
            const unsigned hi_t = __reduce_max_sync(0xffffffffu, t);
            const unsigned mb = __float_as_uint(m);
            const unsigned m_lo = __reduce_max_sync(0xffffffffu, t == lo_t ? mb : 0u);
            const unsigned m_hi = __reduce_max_sync(0xffffffffu, t != lo_t ? mb : 0u);
            if (lane == 0) {
                if (lo_t < (unsigned)T) atomicMax(&R.amax[lo_t], m_lo);
                if (hi_t != lo_t && hi_t < (unsigned)T) atomicMax(&R.amax[hi_t], m_hi);
            }
        }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < ngrp; c += blockDim.x) {
        const int t = c / n8;
        const int sh = p.act_type == NVFP4_MOE_ACT_INT8 ? 0 : pow2_shift_for(__uint_as_float(R.amax[t]));
        float v[8];
        act8(p, S.raw, t, c % n8, v);
        const uint4 pk = pack8_f16(v, sh);
        uint2 *dst = reinterpret_cast<uint2 *>(S.xs + t * ld + 8 * (c % n8));
        dst[0] = make_uint2(pk.x, pk.y);
        dst[1] = make_uint2(pk.z, pk.w);
    }
    if (threadIdx.x < T)
        R.xsc[threadIdx.x] = p.act_type == NVFP4_MOE_ACT_INT8
                                 ? p.act_scale[threadIdx.x]
                                 : exp2i(-pow2_shift_for(__uint_as_float(R.amax[threadIdx.x])));
    if (blockIdx.x == 0) publish_route(p, R);
    // this CTA's stripe of out is cleared for the combine (unless accumulating)
    if (!p.out_add) {
        int za, zb;
        share(T * H / 4, blockIdx.x, gridDim.x, za, zb);
        for (int c = za + threadIdx.x; c < zb; c += blockDim.x)
            reinterpret_cast<float4 *>(p.out)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    // the activations are read and this stripe of out is cleared: phase-2 adds
    // anywhere into out wait for every CTA to get here (out may alias act)
    if (threadIdx.x == 0 && !((p.test_flags & NVFP4_MOE_TEST_DECODE_STALL) && blockIdx.x == 0)) {
        __threadfence();
        atomicAdd(ds + kDsStaged, 1);
    }

    // first weight loads after the staging: the fence above then has no weight
    // loads of its own thread to wait for
    issue_loads<0>(p, item_of<0>(p, R, c1), lane >> 2, lane & 3, c1.r0, c1.r1, buf0);
    run_range<0>(p, R, S, x1, b1, c1, buf0, buf1, 0);

    // phase 2: this CTA's share, split evenly over its warps
    int ca, cb;
    share(n2, blockIdx.x, gridDim.x, ca, cb);
    int a2, b2;
    share(cb - ca, warp, kDecWarps, a2, b2);
    a2 += ca;
    b2 += ca;
    int x2 = a2;
    const Chunk c2 = take_chunk(x2, b2, R2);
    issue_loads<1>(p, item_of<1>(p, R, c2), lane >> 2, lane & 3, c2.r0, c2.r1, buf0);
    const int per_u2 = (H / 16) * R2;
    const int u_lo = ca / per_u2, u_hi = cb > ca ? (cb - 1) / per_u2 : u_lo - 1;
    const int pos_lo = u_hi >= u_lo ? R.uoff[u_lo] : 0;
    const int rows = u_hi >= u_lo ? R.uoff[u_hi + 1] - pos_lo : 0;
    __syncthreads();
    // This CTA's last use of the counts is the wait below; once every CTA has
    // passed it, every count is final (each used expert has down items, so its
    // gate/up items are all finished), and the last CTA to arrive resets them.
    // The arrival is issued right after the wait and its result is consumed at
    // the end, so its round trip hides behind the down work.
    int exit_prev = 0;
    if (threadIdx.x == 0) {
        if (u_hi >= u_lo) {
            bool ok = wait_geq(ds + kDsStaged, gridDim.x, p.status, 101);
            for (int u = u_lo; ok && u <= u_hi; u++) ok = wait_geq(ds + kDsReady + u, I / 8, p.status, 102);
            if (rows > p.dec_hs_rows) latch_status(p.status, NVFP4_MOE_ERR_UNSUPPORTED_DIMS, 103);
            __threadfence();
        }
        exit_prev = atomicAdd(ds + kDsExit, 1);
    }
    __syncthreads();
    {
        const int nrow = min(rows, p.dec_hs_rows), per_row = I / 8;   // 16-byte pieces per h row
        for (int c = threadIdx.x; c < nrow * per_row; c += blockDim.x) {
            const int r = c / per_row, k = c - r * per_row;
            cp_async16(S.hs + (size_t)r * (I + 8) + 8 * k, p.h + (size_t)(pos_lo + r) * I + 8 * k);
        }
        asm volatile("cp.async.commit_group;\n cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();
    if (rows <= p.dec_hs_rows) run_range<1>(p, R, S, x2, b2, c2, buf0, buf1, pos_lo);

    // The next layer's grid may launch once every CTA is here.
    if (threadIdx.x == 0 && exit_prev == (int)gridDim.x - 1) {
        for (int u = 0; u < U; u++) ds[kDsReady + u] = 0;
        ds[kDsStaged] = 0;
        ds[kDsExit] = 0;
    }
    grid_dep_launch();
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// h rows one CTA's phase-2 range can touch: a range of at most
// ceil(U * per_u / G) units touches at most floor(U / G) + 2 used experts, each
// with at most T pairs.
int decode_hs_rows(int T, int K, int E, int grid) {
    const int P = T * K, U_max = P < E ? P : E;
    const int r = (U_max / grid + 2) * T;
    return r < P ? r : P;
}

int decode_grid() { return sm_count(); }

static size_t decode_smem(const Params &p) {
    return (size_t)kSlots * (p.H + 4) * sizeof(__half) + (size_t)p.T * raw_act_bytes(p.act_type, p.H) +
           (size_t)p.dec_hs_rows * (p.I + 8) * sizeof(__half);
}

template <int NPER>
static cudaError_t launch_layer(const Params &p, cudaStream_t s) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(decode_grid());
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = decode_smem(p);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_layer_kernel<NPER>, p);
}

cudaError_t launch_decode(const Params &p, cudaStream_t s) {
    const int n = cdiv(p.E, 32);
    if (n <= 1) return launch_layer<1>(p, s);
    if (n <= 2) return launch_layer<2>(p, s);
    if (n <= 4) return launch_layer<4>(p, s);
    if (n <= 8) return launch_layer<8>(p, s);
    if (n <= 16) return launch_layer<16>(p, s);
    return launch_layer<32>(p, s);
}

cudaError_t decode_init() {
    // dynamic shared memory above 48 KB (the F16 activations grow with H)
    const int big = 200 * 1024;
    const cudaError_t r[] = {
        cudaFuncSetAttribute(decode_layer_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_layer_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_layer_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_layer_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_layer_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_layer_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, big)};
    for (cudaError_t x : r)
        if (x != cudaSuccess) return x;
    return cudaSuccess;
}

}  // namespace nvmoe
