// Decode path (T <= 8): stream each selected expert's 4.5-bit weights once.
//
// The pages keep the quality profile on "canonical FP32 expert decode" ("#1858
// ... strata-safetensors", "What do you want to do?" and the paragraph after
// the measurements) and note that a decode round is bound by moving expert
// bytes ("Strata NVFP4" README, "Limits"). On B200 every expert is resident in
// HBM, so decode is a pure HBM stream whose time is set by how early the weight
// loads start and how many are in flight.
//
// Two kernels, linked by programmatic dependent launch:
//   gate/up: waits for the previous grid (griddepcontrol.wait), then every CTA
//     routes the <= 8 tokens itself (top-k over at most 8 x E logits is a few
//     microseconds of one warp per token), so it knows the selected experts
//     without another kernel or a grid-wide barrier, and starts its weight stream.
//   down: launched as soon as every gate/up CTA has passed its wait; routes again
//     in every CTA, issues its first weight loads, and only then waits for the
//     gate/up grid (whose h it needs), so its weight stream overlaps the gate/up
//     kernel.
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

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kMaxRoundsPerWarp = 4;   // 128-wide K rounds of loads one warp holds per pass
constexpr int kMaxUniq = NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK;  // 128
constexpr int kSlots = NVFP4_MOE_DECODE_MAX_T;

// Number of warps that share one item's K range (1, 2 or 4): each warp takes
// rounds/split consecutive rounds; the partial sums meet in shared memory.
__host__ __device__ inline int k_split(int rounds) {
    if (rounds % 4 == 0 && rounds / 4 <= kMaxRoundsPerWarp) return 4;
    if (rounds % 2 == 0 && rounds / 2 <= kMaxRoundsPerWarp) return 2;
    return rounds <= kMaxRoundsPerWarp ? 1 : 4;
}

// Per-CTA routing state of the decode kernels.
struct DecRoute {
    int ids[kSlots * NVFP4_MOE_MAX_TOPK];
    float w[kSlots * NVFP4_MOE_MAX_TOPK];
    int uniq[kMaxUniq];             // selected experts, ascending
    int upos[kMaxUniq * kSlots];    // pair position of (unique expert, token), -1 if absent
    float uw[kMaxUniq * kSlots];    // routing weight of (unique expert, token)
    unsigned amax[kSlots];          // per-token activation amax (FP32 bits)
    float xsc[kSlots];              // per-token factor that undoes the F16 staging scale
    int U, total;
    int wt[33];
};

// Routes the T <= 8 tokens inside one CTA (identical result in every CTA):
// top-k + weights, per-expert token masks, counts and offsets by one packed
// scan, the unique-expert list and each (expert, token) position and weight.
// emask/cnt: E ints each of dynamic shared memory.
template <int NPER>
__device__ void cta_route(const Params &p, DecRoute &R, int *emask, int *cnt, bool report) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) emask[e] = 0;
    __syncthreads();
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
            atomicOr(&emask[id], 1 << warp);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const int c = __popc(emask[e]);
        cnt[e] = c | ((c != 0) << 16);   // pairs (low 16 bits), used experts (high 16 bits)
    }
    __syncthreads();
    const int both = block_exscan(cnt, p.E, R.wt);
    if (threadIdx.x == 0) {
        R.total = both & 0xFFFF;
        R.U = both >> 16;
    }
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
        if (emask[e]) R.uniq[cnt[e] >> 16] = e;
    for (int i = threadIdx.x; i < kMaxUniq * kSlots; i += blockDim.x) R.upos[i] = -1;
    __syncthreads();
    for (int q = threadIdx.x; q < p.T * p.K; q += blockDim.x) {   // one thread per (token, slot)
        const int t = q / p.K, e = R.ids[q];
        const int u = cnt[e] >> 16;
        R.upos[u * kSlots + t] = (cnt[e] & 0xFFFF) + __popc(emask[e] & ((1 << t) - 1));
        R.uw[u * kSlots + t] = R.w[q];
    }
    __syncthreads();
}

// The routing results a forward call leaves in the workspace (and the optional
// debug copies); written by CTA 0 after the previous grid has finished.
__device__ void publish_route(const Params &p, const DecRoute &R, const int *emask, const int *cnt) {
    for (int q = threadIdx.x; q < p.T * p.K; q += blockDim.x) {
        const int t = q / p.K, e = R.ids[q];
        const int pos = (cnt[e] & 0xFFFF) + __popc(emask[e] & ((1 << t) - 1));
        p.ids[q] = e;
        p.wts[q] = R.w[q];
        p.perm[pos] = q;
        p.inv[q] = pos;
        p.ptok[pos] = t;
        p.pw[pos] = R.w[q];
        if (p.dbg_ids) p.dbg_ids[q] = e;
        if (p.dbg_w) p.dbg_w[q] = R.w[q];
        if (p.dbg_perm) p.dbg_perm[pos] = q;
    }
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
        const int off = e < p.E ? (cnt[e] & 0xFFFF) : R.total;
        p.offsets[e] = off;
        if (p.dbg_offsets) p.dbg_offsets[e] = off;
        if (e < p.E) {
            const int c = __popc(emask[e]);
            p.counts[e] = c;
            if (p.dbg_counts) p.dbg_counts[e] = c;
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

template <int MODE>
__device__ inline ItemRef item_ref(const Params &p, const DecRoute &R, int item, int items) {
    ItemRef r{0, 0, 0, item < items};
    if (r.valid) {
        const int per_u = MODE == 0 ? p.I / 8 : p.H / 16;
        r.u = item / per_u;
        r.m0 = (item % per_u) * (MODE == 0 ? 8 : 16);
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

// Grid-wide barrier for a cooperatively launched grid (all CTAs co-resident),
// used once per kernel. Each CTA reads the generation word, then arrives on the
// count; the last to arrive advances the generation (which the others poll) and
// only then resets the count, so the release costs two dependent atomics and the
// words (in the handle's device status block) are ready for the next launch. The
// wait is bounded: after `limit_ns` it latches NVFP4_MOE_ERR_TIMEOUT and returns.
__device__ inline void grid_barrier_once(int32_t *status, uint64_t limit_ns = 200000000ull) {
    unsigned *gen = reinterpret_cast<unsigned *>(status + kStatusBarGen);
    unsigned *count = reinterpret_cast<unsigned *>(status + kStatusBarTop);
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile unsigned *vgen = gen;
        const unsigned my_gen = *vgen;
        __threadfence();
        if (atomicAdd(count, 1u) + 1u == gridDim.x) {
            atomicAdd(gen, 1u);
            atomicExch(count, 0u);
        } else {
            const uint64_t t0 = globaltimer();
            while (*vgen == my_gen) {
                __nanosleep(20);
                if (globaltimer() - t0 > limit_ns) {
                    latch_status(status, NVFP4_MOE_ERR_TIMEOUT, 100);
                    break;
                }
            }
        }
        __threadfence();
    }
    __syncthreads();
}

struct DecSmem {
    float *red;     // [8 warps][32][4] split-K partial sums
    __half *xs;     // [8 token slots][H+4] F16 activations
    uint8_t *raw;   // [T][H] raw BF16 / int8 activations (cp.async at kernel start)
};

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

// The weight-streaming passes of one projection over this CTA's share of the
// items. MODE 0: gate/up + SwiGLU; item = (unique expert u, 8 intermediate rows):
// A rows g are gate rows, rows g+8 the up rows of the same intermediate index,
// so each thread ends with g and u of the same (row, token) pair. MODE 1: down +
// weighted combine; item = (unique expert u, 16 hidden rows); B = h of the pairs
// (token, u), zero for tokens not routed to u. Each pass covers kDecWarps/split
// items; the next pass's loads are issued before the current pass computes (two
// register buffers). On entry buf0 already holds this CTA's first pass.
template <int MODE>
__device__ inline void run_passes(const Params &p, const DecRoute &R, const DecSmem &S,
                                  PassBuf &buf0, PassBuf &buf1) {
    const int H = p.H, I = p.I, T = p.T;
    const int rounds = (MODE == 0 ? H : I) / 128;
    const int split = k_split(rounds);
    const int rpw = cdiv(rounds, split);
    const int ipc = kDecWarps / split;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int items = R.U * ((MODE == 0 ? I : H) / (MODE == 0 ? 8 : 16));
    const int item_l = warp / split, part = warp % split;
    const int r_begin = part * rpw, r_end = min(rounds, r_begin + rpw);
    const int stride = gridDim.x * ipc;
    const int ld = H + 4;
    const __half *xrow = S.xs + g * ld + 32 * q;
    int base = blockIdx.x * ipc;
    ItemRef cur = item_ref<MODE>(p, R, base + item_l, items);

    auto pass_step = [&](PassBuf &b, PassBuf &nb) {
        const ItemRef nxt = item_ref<MODE>(p, R, base + stride + item_l, items);
        issue_loads<MODE>(p, nxt, g, q, r_begin, r_end, nb);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (cur.valid) {
            const int mypos = (MODE == 1 && g < T) ? R.upos[cur.u * kSlots + g] : -1;
            const __half *hrow = p.h + (size_t)(mypos < 0 ? 0 : mypos) * I + 32 * q;
#pragma unroll
            for (int j = 0; j < kMaxRoundsPerWarp; j++) {
                const int r = r_begin + j;
                if (r < r_end) {
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
        }
        if (split > 1) {
            *reinterpret_cast<float4 *>(S.red + (warp * 32 + lane) * 4) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
            __syncthreads();
            if (part == 0) {
                for (int w2 = 1; w2 < split; w2++) {
                    const float4 o = *reinterpret_cast<const float4 *>(S.red + ((warp + w2) * 32 + lane) * 4);
                    acc[0] += o.x;
                    acc[1] += o.y;
                    acc[2] += o.z;
                    acc[3] += o.w;
                }
            }
            __syncthreads();
        }
        if (part == 0 && cur.valid) {
            if (MODE == 0) {
                const float sgl = p.gate_global[cur.e], sul = p.up_global[cur.e];
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const int tok = 2 * q + c;
                    const int pos = tok < T ? R.upos[cur.u * kSlots + tok] : -1;
                    if (pos >= 0) {
                        const float gv = acc[c] * sgl * R.xsc[tok], uv = acc[2 + c] * sul * R.xsc[tok];
                        p.h[(size_t)pos * I + cur.m0 + g] = __float2half_rn(silu(gv) * uv);
                    }
                }
            } else {
                const float sd = p.down_global[cur.e];
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const int tok = 2 * q + c;
                    if (tok < T && R.upos[cur.u * kSlots + tok] >= 0) {
                        const float w = R.uw[cur.u * kSlots + tok] * sd;
                        atomicAdd(p.out + (size_t)tok * H + cur.m0 + g, acc[c] * w);
                        atomicAdd(p.out + (size_t)tok * H + cur.m0 + g + 8, acc[2 + c] * w);
                    }
                }
            }
        }
        cur = nxt;
        base += stride;
    };
    while (base < items) {
        pass_step(buf0, buf1);
        if (base >= items) break;
        pass_step(buf1, buf0);
    }
}

template <int MODE>
__device__ inline void first_loads(const Params &p, const DecRoute &R, PassBuf &b) {
    const int rounds = (MODE == 0 ? p.H : p.I) / 128;
    const int split = k_split(rounds);
    const int rpw = cdiv(rounds, split);
    const int ipc = kDecWarps / split;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int items = R.U * ((MODE == 0 ? p.I : p.H) / (MODE == 0 ? 8 : 16));
    const int part = warp % split, r_begin = part * rpw;
    const ItemRef it = item_ref<MODE>(p, R, blockIdx.x * ipc + warp / split, items);
    issue_loads<MODE>(p, it, lane >> 2, lane & 3, r_begin, min(rounds, r_begin + rpw), b);
}

// The whole decode layer in one cooperatively launched grid: every CTA routes
// the <= 8 tokens itself, stages the F16 activations, streams its share of the
// gate/up weights (SwiGLU into h), issues its first down-projection loads, and
// after one grid-wide barrier (h complete, out cleared) streams its share of the
// down weights with the weighted combine.
template <int NPER>
__global__ void __launch_bounds__(kDecThreads, 2) decode_layer_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ DecRoute R;
    const int H = p.H, T = p.T;
    DecSmem S;
    S.red = reinterpret_cast<float *>(dsm);
    int *emask = reinterpret_cast<int *>(dsm + kDecWarps * 32 * 4 * sizeof(float));
    int *cnt = emask + p.E;
    S.xs = reinterpret_cast<__half *>(cnt + p.E);
    S.raw = reinterpret_cast<uint8_t *>(S.xs + kSlots * (H + 4));
    const int ld = H + 4;

    // the activations first: their loads are then not queued behind the weights'
    const int raw_bytes = T * raw_act_bytes(p.act_type, H);
    for (int c = threadIdx.x; c < raw_bytes / 16; c += blockDim.x)
        cp_async16(S.raw + 16 * c, static_cast<const uint8_t *>(p.act) + 16 * c);
    asm volatile("cp.async.commit_group;" ::: "memory");

    cta_route<NPER>(p, R, emask, cnt, blockIdx.x == 0);
    PassBuf buf0, buf1;
    first_loads<0>(p, R, buf0);

    // per-token amax -> power-of-two shift -> F16 activations in shared memory
    // (token slots past T are zeros); every load of x is issued before its use
    const int n8 = H / 8;
    for (int c = threadIdx.x; c < (kSlots - T) * n8; c += blockDim.x) {
        uint2 *dst = reinterpret_cast<uint2 *>(S.xs + (T + c / n8) * ld + 8 * (c % n8));
        dst[0] = make_uint2(0, 0);
        dst[1] = make_uint2(0, 0);
    }
    if (threadIdx.x < kSlots) R.amax[threadIdx.x] = 0u;
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // two passes over the shared raw copy (global memory for FP32 input): the
    // per-token amax (reduced per warp, one shared atomic per warp and token),
    // then the shifted F16 values. Loop bounds are whole warps for the shuffles.
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
            if ((threadIdx.x & 31) == 0) {
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
    if (blockIdx.x == 0) publish_route(p, R, emask, cnt);
    // out is cleared for the combine before the grid barrier below; act never
    // aliases out in this mode (only an accumulating call may pass act == out)
    if (!p.out_add)
        for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < T * H / 4; c += gridDim.x * blockDim.x)
            reinterpret_cast<float4 *>(p.out)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();

    run_passes<0>(p, R, S, buf0, buf1);
    first_loads<1>(p, R, buf0);     // down weights in flight while the grid catches up
    grid_barrier_once(p.status);    // h complete, out cleared
    run_passes<1>(p, R, S, buf0, buf1);
}

static int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

static size_t decode_smem(const Params &p) {
    return kDecWarps * 32 * 4 * sizeof(float) + 2 * (size_t)p.E * sizeof(int) +
           (size_t)8 * (p.H + 4) * sizeof(__half) + (size_t)p.T * raw_act_bytes(p.act_type, p.H);
}

template <int NPER>
static cudaError_t launch_layer(const Params &p, cudaStream_t s) {
    const size_t smem = decode_smem(p);
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_layer_kernel<NPER>,
                                                                  kDecThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int U_max = min(p.T * p.K, p.E);
    const int need = max(cdiv(U_max * (p.I / 8), kDecWarps / k_split(p.H / 128)),
                         cdiv(U_max * (p.H / 16), kDecWarps / k_split(p.I / 128)));
    const int grid = max(1, min(min(per_sm, 2) * sm_count(), need));
    Params pp = p;
    void *args[] = {&pp};
    return cudaLaunchCooperativeKernel((const void *)decode_layer_kernel<NPER>, dim3(grid),
                                       dim3(kDecThreads), args, smem, s);
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
