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
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        const int m = emask[e];
        if (!m) continue;
        const int u = cnt[e] >> 16, off = cnt[e] & 0xFFFF;
        R.uniq[u] = e;
        for (int t = 0; t < kSlots; t++) {
            int pos = -1;
            float wt = 0.0f;
            if ((m >> t) & 1) {
                pos = off + __popc(m & ((1 << t) - 1));
                for (int j = 0; j < p.K; j++)
                    if (R.ids[t * p.K + j] == e) wt = R.w[t * p.K + j];
            }
            R.upos[u * kSlots + t] = pos;
            R.uw[u * kSlots + t] = wt;
        }
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

// MODE 0: gate/up + SwiGLU. Item = (unique expert u, 8 intermediate rows): A
//   rows g are gate rows, rows g+8 the up rows of the same intermediate index, so
//   each thread ends with g and u of the same (row, token) pair.
// MODE 1: down + weighted combine. Item = (unique expert u, 16 hidden rows); the
//   B operand is h of the pairs (token, u), zero for tokens not routed to u.
// Persistent CTAs: each pass covers kDecWarps/split items; the weight loads of
// the next pass are issued before the current pass computes (two register
// buffers), so every warp keeps its HBM stream going across passes.
template <int MODE, int NPER>
__global__ void __launch_bounds__(kDecThreads, 2) decode_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ DecRoute R;
    // gate/up may start before the previous grid (for instance the one that wrote
    // the router logits) has finished: it waits before reading any input, and
    // only then lets its dependent (the down kernel) launch. The down kernel's
    // predecessor is this gate/up grid, which writes none of the routing inputs
    // or weights, so it routes and starts its weight stream before waiting.
    if (MODE == 0) grid_dep_wait();
    grid_dep_launch();
    const int H = p.H, I = p.I, T = p.T;
    float *red = reinterpret_cast<float *>(dsm);                               // [8][32][4]
    int *emask = reinterpret_cast<int *>(dsm + kDecWarps * 32 * 4 * sizeof(float));
    int *cnt = emask + p.E;
    __half *xs = reinterpret_cast<__half *>(cnt + p.E);                        // [8][H+4] (MODE 0)
    const int ld = H + 4;

    cta_route<NPER>(p, R, emask, cnt, blockIdx.x == 0);

    const int Kd = MODE == 0 ? H : I;
    const int rounds = Kd / 128;
    const int split = k_split(rounds);
    const int rpw = cdiv(rounds, split);
    const int ipc = kDecWarps / split;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int items = R.U * ((MODE == 0 ? I : H) / (MODE == 0 ? 8 : 16));
    const int item_l = warp / split, part = warp % split;
    const int r_begin = part * rpw, r_end = min(rounds, r_begin + rpw);
    const int stride = gridDim.x * ipc;

    PassBuf buf0, buf1;
    int base = blockIdx.x * ipc;
    ItemRef cur = item_ref<MODE>(p, R, base + item_l, items);
    issue_loads<MODE>(p, cur, g, q, r_begin, r_end, buf0);

    // down: from here on it reads h, written by the gate/up grid
    if (MODE == 1) grid_dep_wait();
    if (MODE == 0) {
        // per-token amax -> power-of-two shift -> F16 activations of the 8 token
        // slots (zeros past T) in shared memory
        if (threadIdx.x < kSlots) R.amax[threadIdx.x] = 0u;
        __syncthreads();
        const int n8 = H / 8;
        if (p.act_type != NVFP4_MOE_ACT_INT8) {
            for (int c = threadIdx.x; c < T * n8; c += blockDim.x) {
                float v[8];
                load_act8(p, c / n8, c % n8, v);
                float m = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; j++) m = fmaxf(m, fabsf(v[j]));
                atomicMax(&R.amax[c / n8], __float_as_uint(m));
            }
        }
        __syncthreads();
        for (int c = threadIdx.x; c < kSlots * n8; c += blockDim.x) {
            const int t = c / n8, k8 = c % n8;
            uint4 pk = make_uint4(0, 0, 0, 0);
            if (t < T) {
                const int sh = p.act_type == NVFP4_MOE_ACT_INT8 ? 0 : pow2_shift_for(__uint_as_float(R.amax[t]));
                float v[8];
                load_act8(p, t, k8, v);
                pk = pack8_f16(v, sh);
            }
            uint2 *d = reinterpret_cast<uint2 *>(xs + t * ld + 8 * k8);
            d[0] = make_uint2(pk.x, pk.y);
            d[1] = make_uint2(pk.z, pk.w);
        }
        if (threadIdx.x < T)
            R.xsc[threadIdx.x] = p.act_type == NVFP4_MOE_ACT_INT8
                                     ? p.act_scale[threadIdx.x]
                                     : exp2i(-pow2_shift_for(__uint_as_float(R.amax[threadIdx.x])));
        if (blockIdx.x == 0) publish_route(p, R, emask, cnt);
        if (!p.out_add)   // clear out for the down kernel's reductions, split over the grid
            for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < T * H / 4; c += gridDim.x * blockDim.x)
                reinterpret_cast<float4 *>(p.out)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        __syncthreads();
    }
    const __half *xrow = xs + g * ld + 32 * q;

    // one pass: compute from b while the next pass's loads fill nb
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
            *reinterpret_cast<float4 *>(red + (warp * 32 + lane) * 4) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
            __syncthreads();
            if (part == 0) {
                for (int w2 = 1; w2 < split; w2++) {
                    const float4 o = *reinterpret_cast<const float4 *>(red + ((warp + w2) * 32 + lane) * 4);
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

static int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int MODE, int NPER>
static void launch_one(const Params &p, cudaStream_t s) {
    const int U_max = min(p.T * p.K, p.E);
    const int rounds = (MODE == 0 ? p.H : p.I) / 128;
    const int ipc = kDecWarps / k_split(rounds);
    const int items = U_max * (MODE == 0 ? p.I / 8 : p.H / 16);
    const size_t smem = kDecWarps * 32 * 4 * sizeof(float) + 2 * (size_t)p.E * sizeof(int) +
                        (MODE == 0 ? (size_t)8 * (p.H + 4) * sizeof(__half) : 0);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(max(1, min(2 * sm_count(), cdiv(items, ipc))));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, decode_kernel<MODE, NPER>, p);
}

#define DEC_NPER_SWITCH(E, MODE)                                                  \
    do {                                                                          \
        const int _n = cdiv((E), 32);                                             \
        if (_n <= 1) launch_one<MODE, 1>(p, s);                                   \
        else if (_n <= 2) launch_one<MODE, 2>(p, s);                              \
        else if (_n <= 4) launch_one<MODE, 4>(p, s);                              \
        else if (_n <= 8) launch_one<MODE, 8>(p, s);                              \
        else if (_n <= 16) launch_one<MODE, 16>(p, s);                            \
        else launch_one<MODE, 32>(p, s);                                          \
    } while (0)

void launch_decode_gateup(const Params &p, cudaStream_t s) { DEC_NPER_SWITCH(p.E, 0); }
void launch_decode_down(const Params &p, cudaStream_t s) { DEC_NPER_SWITCH(p.E, 1); }

cudaError_t decode_init() {
    // dynamic shared memory above 48 KB for the gate/up kernel at large H
    const int big = 200 * 1024;
#define DEC_ATTR(M, N) cudaFuncSetAttribute(decode_kernel<M, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, big)
    const cudaError_t r[] = {DEC_ATTR(0, 1), DEC_ATTR(0, 2), DEC_ATTR(0, 4), DEC_ATTR(0, 8),
                             DEC_ATTR(0, 16), DEC_ATTR(0, 32), DEC_ATTR(1, 1), DEC_ATTR(1, 2),
                             DEC_ATTR(1, 4), DEC_ATTR(1, 8), DEC_ATTR(1, 16), DEC_ATTR(1, 32)};
#undef DEC_ATTR
    for (cudaError_t x : r)
        if (x != cudaSuccess) return x;
    return cudaSuccess;
}

}  // namespace nvmoe
