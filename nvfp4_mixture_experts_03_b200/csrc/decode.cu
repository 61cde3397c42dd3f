// Decode path (T <= 8): stream each selected expert's 4.5-bit weights once.
//
// The pages keep the quality profile on "canonical FP32 expert decode" ("#1858
// ... strata-safetensors", "What do you want to do?" and the paragraph after
// the measurements) and note that a decode round is bound by moving expert
// bytes ("Strata NVFP4" README, "Limits"). On B200 every expert is resident in
// HBM, so decode is a pure HBM stream whose time is set by how early the weight
// copies start, how many bytes are in flight and how evenly they are spread.
//
// One kernel per layer, one CTA per SM (16 consumer warps + 2 producer warps),
// launched with programmatic dependent launch:
//   routing: every CTA routes the <= 8 tokens itself (warp top-k per token, then
//     the <= 128 (token, slot) pairs ranked by (expert, token)), so no CTA waits
//     for another before its weight stream starts;
//   work: phase-1 items (used expert u, 8 intermediates: 8 gate + 8 up rows, all
//     of K = H) and phase-2 items (u, 16 hidden rows, all of K = I) are cut into
//     equal contiguous ranges, one range of each per CTA;
//   producer warps: as soon as routing is done, one copies the CTA's phase-1
//     items and the other its phase-2 items into two shared-memory rings with 1-D
//     bulk copies (each item's code rows and scale rows are contiguous blocks
//     of each projection), so the down weights stream in while gate/up computes;
//   consumer warps: each warp owns fixed 128-wide K rounds of an item, and holds
//     the activations (phase 1) or the expert's h rows (phase 2) of those rounds
//     in registers as mma.sync B fragments. A group of warps covers one item's K;
//     their FP32 partial sums meet in shared memory and are added in a fixed warp
//     order. Phase 1 ends in SwiGLU and the F16 h row; each finished item counts
//     towards its expert's ready count. Phase 2 waits for its expert's count,
//     writes w * s_d * y per pair as FP32 rows, and the CTA that completes a block
//     of 16 hidden rows (one item per used expert) adds each token's K rows in the
//     fixed order j = 0..K-1 into out. No floating-point atomics: the output is
//     the same bits on every run.
// Cross-CTA waits (expert ready counts, the count of CTAs that have read the
// activations, which out may alias) are bounded; the last CTA to finish resets
// the counters for the next launch.
// Arithmetic: each weight is decoded exactly to F16 (E2M1 -> F16 conversion
// times its E4M3 group scale: at most 6 significant bits) and fed to mma.sync
// m16n8k16 with the token slots as N, FP32 accumulation; the tensor scale and
// the per-token activation scale are applied to the FP32 result.
//
// Fragment mapping (m16n8k16, A row-major, B col-major): thread (g = lane/4,
// q = lane%4) holds A rows g and g+8; per 128-wide K round it reads 16
// contiguous code bytes of each row (byte offset 64*r + 16*q). Mma step s of
// round r uses physical K 128r + 32q + 4s + {0,1,2,3} for logical K {2q, 2q+1,
// 2q+8, 2q+9}; the B fragments use the same permutation, so every dot product
// is the plain one. H and I need only be multiples of 32: a 32-wide piece of a
// round past the end is zero on both sides.
#include "common.cuh"
#include "route_common.cuh"

namespace nvmoe {

// Timeline marks for profiling builds (compiled with NVMOE_DEC_TRACE): the
// global timer per CTA at a few points of the layer; nothing otherwise.
#ifdef NVMOE_DEC_TRACE
__device__ unsigned long long g_dec_trace[1024][8];
#define DEC_MARK(i) (g_dec_trace[blockIdx.x][(i)] = globaltimer())
#else
#define DEC_MARK(i) ((void)0)
#endif

__device__ inline void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

constexpr int kDecCW = 16;                          // consumer warps
constexpr int kDecThreads = (kDecCW + 2) * 32;      // + two producer warps (one per ring)
constexpr int kMaxRW = 3;                           // K rounds of B fragments a warp holds
constexpr int kMaxPairs = NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK;  // 128
constexpr int kSlots = NVFP4_MOE_DECODE_MAX_T;
constexpr int kPartBytes = kDecCW * 2 * 32 * 16;    // partial sums: [warp][2 buffers][lane] float4
constexpr int kBarConsumers = 15;                   // named barrier over the 16 consumer warps
constexpr uint64_t kDecWaitNs = 200000000ull;
constexpr uint64_t kDecDrainNs = 200000000ull;
constexpr int kDecSmemBudget = 208 * 1024;          // dynamic shared memory the plan may use (+ about 12 KB static)

// Warps per item for a projection of NR K rounds: the fewest (2, 4, 8 or 16)
// that leave each warp at most kMaxRW rounds; 0 when NR is too large.
__host__ __device__ inline int dec_group_warps(int nr) {
    for (int wg = 2; wg <= kDecCW; wg *= 2)
        if (cdiv(nr, wg) <= kMaxRW) return wg;
    return 0;
}

// Per-CTA routing state of the decode kernel.
struct DecRoute {
    int ids[kMaxPairs];
    float w[kMaxPairs];
    int pos[kMaxPairs];             // position of pair q (grouped by expert, then token)
    int sorted_e[kMaxPairs];        // expert at each position
    int uniq[kMaxPairs];            // used experts, ascending
    int upos[kMaxPairs * kSlots];   // pair position of (used expert, token), -1 if absent
    float uw[kMaxPairs * kSlots];   // routing weight of (used expert, token)
    unsigned amax[kSlots];          // per-token activation amax (FP32 bits)
    int wtot[33];                   // block scan scratch
    int U;
};

// Routes the T <= 8 tokens inside one CTA (identical result in every CTA).
// Positions come from counting, not sorting: per expert, the number of pairs and
// a bitmask of the tokens that chose it (one shared int: count in bits 0..15,
// token t in bit 16 + t -- a token names an expert at most once); one block-wide
// exclusive scan over the experts gives each expert's first position and its
// index among the used experts; a pair's position is its expert's first position
// plus the number of earlier tokens in the mask. `ex` and `sc` are E ints of
// shared scratch each.
template <int NPER>
__device__ void cta_route(const Params &p, DecRoute &R, bool report, int *ex, int *sc) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.T * p.K, E = p.E;
    for (int i = threadIdx.x; i < kMaxPairs * kSlots; i += blockDim.x) R.upos[i] = -1;
    for (int i = threadIdx.x; i < E; i += blockDim.x) ex[i] = 0;
    if (threadIdx.x < kSlots) R.amax[threadIdx.x] = 0u;
    __syncthreads();
    if (warp < p.T) {
        int id;
        float w;
        if (p.logits) {
            bool finite;
            warp_topk<NPER>(p.logits + (size_t)warp * E, E, p.K, lane, id, w, finite);
            if (!finite && report && lane == 0) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, warp);
        } else {
            const bool ok = warp_given(p.in_ids + (size_t)warp * p.K, p.in_w + (size_t)warp * p.K,
                                       E, p.K, lane, id, w);
            if (!ok && report && lane == 0) latch_status(p.status, NVFP4_MOE_ERR_BAD_ROUTING, warp);
        }
        if (lane < p.K) {
            R.ids[warp * p.K + lane] = id;
            R.w[warp * p.K + lane] = w;
            atomicAdd(&ex[id], 1 + (1 << (16 + warp)));
        }
    }
    __syncthreads();
    // pairs before each expert (bits 0..15) and used experts before it (16..)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int n = ex[e] & 0xFFFF;
        sc[e] = n | (n ? 1 << 16 : 0);
    }
    __syncthreads();
    const int total = block_exscan(sc, E, R.wtot);
    if (threadIdx.x < P) {
        const int q = threadIdx.x, e = R.ids[q], t = q / p.K;
        const int first = sc[e] & 0xFFFF, u = sc[e] >> 16;
        const int within = __popc(((unsigned)ex[e] >> 16) & ((1u << t) - 1u));
        const int rank = first + within;
        R.pos[q] = rank;
        R.sorted_e[rank] = e;
        R.upos[u * kSlots + t] = rank;
        R.uw[u * kSlots + t] = R.w[q];
        if (within == 0) R.uniq[u] = e;
    }
    if (threadIdx.x == 0) R.U = total >> 16;
    __syncthreads();
}

// The routing results a forward call leaves in the workspace (and the optional
// debug copies); written by CTA 0 at its end. offsets[e] = pairs with an expert
// below e, found by binary search in the expert-sorted positions.
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
    auto lower = [&](int e) {   // first position whose expert is >= e
        int lo = 0, hi = P;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (R.sorted_e[mid] < e) lo = mid + 1; else hi = mid;
        }
        return lo;
    };
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
        const int before = lower(e);
        p.offsets[e] = before;
        if (p.dbg_offsets) p.dbg_offsets[e] = before;
        if (e < p.E) {
            const int at = lower(e + 1) - before;
            p.counts[e] = at;
            if (p.dbg_counts) p.dbg_counts[e] = at;
        }
    }
    if (threadIdx.x == 0) p.cnt[kCntUniq] = R.U;
}

// Eight mma steps of one 128-wide K round: A rows (g: ca, g+8: cb) as 16 code
// bytes each with their two group scales; B fragments of the round in bx.
__device__ inline void round_mma(float (&acc)[4], const uint4 &ca, const uint4 &cb, uint32_t sa,
                                 uint32_t sb, const uint4 (&bx)[4]) {
    const uint32_t sa0 = e4m3_to_f16x2_bcast(sa & 0xFF), sa1 = e4m3_to_f16x2_bcast(sa >> 8);
    const uint32_t sb0 = e4m3_to_f16x2_bcast(sb & 0xFF), sb1 = e4m3_to_f16x2_bcast(sb >> 8);
    const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w}, wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
    for (int w = 0; w < 4; w++) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        e2m1x8_to_f16(wa[w], a0, a1, a2, a3);   // bytes 4w..4w+3 of row g
        e2m1x8_to_f16(wb[w], b0, b1, b2, b3);   // same bytes of row g+8
        const uint32_t s_a = w < 2 ? sa0 : sa1, s_b = w < 2 ? sb0 : sb1;
        const uint4 &x = bx[w];                 // steps 2w and 2w+1
        mma_16816(acc, hmul2(a0, s_a), hmul2(b0, s_b), hmul2(a1, s_a), hmul2(b1, s_b), x.x, x.y);
        mma_16816(acc, hmul2(a2, s_a), hmul2(b2, s_b), hmul2(a3, s_a), hmul2(b3, s_b), x.z, x.w);
    }
}

// Code bytes and scales of A rows `rowa` and `rowb` for round r of an item held
// in a ring slot: codes [16 rows][kb] bytes, then scales [16 rows][kb/8]; the
// 16-byte pieces of the round past a row's end (kb = K/2 bytes) are zero.
__device__ inline void slot_round(const uint8_t *slot, int kb, int rowa, int rowb, int r, int q,
                                  uint4 &ca, uint4 &cb, uint32_t &sa, uint32_t &sb) {
    const int off = 64 * r + 16 * q;
    if (off < kb) {
        ca = *reinterpret_cast<const uint4 *>(slot + (size_t)rowa * kb + off);
        cb = *reinterpret_cast<const uint4 *>(slot + (size_t)rowb * kb + off);
        const uint8_t *sc = slot + 16 * (size_t)kb;
        const int soff = 8 * r + 2 * q, sk = kb / 8;
        sa = *reinterpret_cast<const unsigned short *>(sc + rowa * sk + soff);
        sb = *reinterpret_cast<const unsigned short *>(sc + rowb * sk + soff);
    } else {
        ca = cb = make_uint4(0, 0, 0, 0);
        sa = sb = 0;
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar` (bytes
// counted by the barrier's transaction count). Both addresses 16-byte aligned,
// size a multiple of 16. No multicast.
__device__ inline void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ inline void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Warp-uniform bounded mbarrier wait of the consumers.
__device__ inline bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int32_t *status,
                                 int where) {
    const bool ok = mbar_wait(bar, parity, abort, status, where, kDecWaitNs);
    return __all_sync(0xffffffffu, ok);
}

// This thread's 32 activations of token t at K offsets k0..k0+31 (k0 < H) as raw
// bits: BF16 in all four words (FP32 input rounded to BF16 on load), int8 in the
// first two.
__device__ inline void load_x32(const Params &p, int t, int k0, uint4 (&v)[4]) {
    const size_t off = (size_t)t * p.H + k0;
    if (p.act_type == NVFP4_MOE_ACT_BF16) {
        const uint4 *s = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.act) + off);
#pragma unroll
        for (int i = 0; i < 4; i++) v[i] = __ldg(s + i);
    } else if (p.act_type == NVFP4_MOE_ACT_INT8) {
        const uint4 *s = reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(p.act) + off);
        v[0] = __ldg(s);
        v[1] = __ldg(s + 1);
        v[2] = v[3] = make_uint4(0, 0, 0, 0);
    } else {
        // out may alias act (residual stream): plain loads, not the read-only path
        const float4 *s = reinterpret_cast<const float4 *>(static_cast<const float *>(p.act) + off);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float4 a = s[2 * i], b = s[2 * i + 1];
            const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; j++)
                w[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * j])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2 * j + 1])) << 16);
            v[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

__device__ inline float raw_amax(const uint4 (&v)[4]) {   // BF16 words
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            m = fmaxf(m, fabsf(__uint_as_float(w[j] << 16)));
            m = fmaxf(m, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
        }
    }
    return m;
}

// Raw activations -> F16 B fragments in place: BF16 scaled by 2^sh (exact), or
// int8 codes (exact in F16).
__device__ inline void to_f16_frags(bool int8, int sh, uint4 (&v)[4]) {
    if (int8) {
        const uint32_t w[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; j++) f[j] = (float)(int8_t)(w[2 * i + (j >> 2)] >> (8 * (j & 3)));
            v[i] = pack8_f16(f, 0);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            float f[8];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                f[2 * j] = __uint_as_float(w[j] << 16);
                f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
            v[i] = pack8_f16(f, sh);
        }
    }
}

// Per-token factors from the routing state: the one that undoes the F16 staging
// of token t's activations (2^-shift, or its int8 scale), and the exponent by
// which its h values are stored (h_exp_for).
__device__ inline float token_xscale(const Params &p, const DecRoute &R, int t) {
    return p.act_type == NVFP4_MOE_ACT_INT8 ? __ldg(p.act_scale + t)
                                            : exp2i(-pow2_shift_for(__uint_as_float(R.amax[t])));
}
__device__ inline int token_hexp(const Params &p, const DecRoute &R, int t) {
    return h_exp_for(p.act_type == NVFP4_MOE_ACT_INT8 ? 127.0f * __ldg(p.act_scale + t)
                                                      : __uint_as_float(R.amax[t]));
}

// Non-blocking release increment: orders this thread's earlier writes (and those
// it has synchronised with) before the count changes; the thread does not wait.
__device__ inline void red_release_add(int32_t *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ inline int ld_acquire(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until *word >= target (one thread, acquire); latches TIMEOUT on
// give-up.
__device__ inline bool wait_geq(const int32_t *word, int target, int32_t *status, int where) {
    if (ld_acquire(word) >= target) return true;
    const uint64_t t0 = globaltimer();
    while (ld_acquire(word) < target) {
        __nanosleep(32);
        if (globaltimer() - t0 > kDecWaitNs) {
            latch_status(status, NVFP4_MOE_ERR_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

// The group's partial sums of an item, added in warp order (deterministic).
__device__ inline float4 group_sum(const float4 *part, int w0, int wg, int buf, int lane) {
    float4 s = part[((size_t)w0 * 2 + buf) * 32 + lane];
    for (int w = 1; w < wg; w++) {
        const float4 o = part[((size_t)(w0 + w) * 2 + buf) * 32 + lane];
        s.x += o.x;
        s.y += o.y;
        s.z += o.z;
        s.w += o.w;
    }
    return s;
}

template <int NPER>
__global__ void __launch_bounds__(kDecThreads, 1) decode_layer_kernel(Params p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ DecRoute R;
    __shared__ int s_abort, s_ok;
    const int H = p.H, I = p.I, T = p.T, K = p.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, q = lane & 3;
    const int N1 = p.dec_n1, N2 = p.dec_n2;
    const int S1 = 9 * H, S2 = 9 * I;             // bytes of one phase-1 / phase-2 item
    const int NR1 = cdiv(H, 128), NR2 = cdiv(I, 128);
    const int WG1 = dec_group_warps(NR1), WG2 = dec_group_warps(NR2);
    float4 *part = reinterpret_cast<float4 *>(dsm);
    uint8_t *ringA = dsm + kPartBytes;
    uint8_t *ringB = ringA + (size_t)N1 * S1;
    uint64_t *full = reinterpret_cast<uint64_t *>(ringB + (size_t)N2 * S2);
    uint64_t *empty = full + N1 + N2;
    volatile int *abort = &s_abort;
    int32_t *ds = p.dstate;

    // Shared memory only before the dependency wait.
    if (threadIdx.x == 0) {
        for (int s = 0; s < N1 + N2; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], s < N1 ? WG1 : WG2);
        }
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Everything this layer reads may come from the previous kernel in the stream.
    grid_dep_wait();
    if (threadIdx.x == 0) DEC_MARK(0);

    // Consumers: this warp's phase-1 activations first, so their loads are in
    // flight while the CTA routes.
    const int wi1 = warp % WG1, g1 = warp / WG1;
    uint4 bx[kMaxRW][4];
    if (warp < kDecCW) {
#pragma unroll
        for (int kk = 0; kk < kMaxRW; kk++) {
            const int k0 = 128 * (wi1 + kk * WG1) + 32 * q;
            if (gq < T && k0 < H) {
                load_x32(p, gq, k0, bx[kk]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++) bx[kk][i] = make_uint4(0, 0, 0, 0);
            }
        }
    }

    // routing scratch: the partial-sum buffers, unused until phase 1
    cta_route<NPER>(p, R, blockIdx.x == 0, reinterpret_cast<int *>(dsm),
                    reinterpret_cast<int *>(dsm) + 1024);
    if (threadIdx.x == 0) DEC_MARK(1);
    const int U = R.U;
    const int per1 = I / 8, per2 = H / 16;        // items per used expert
    const int n1 = U * per1, n2 = U * per2;
    const int G = gridDim.x, c = blockIdx.x;
    const int a1 = (int)((long long)n1 * c / G), b1 = (int)((long long)n1 * (c + 1) / G);
    const int a2 = (int)((long long)n2 * c / G), b2 = (int)((long long)n2 * (c + 1) / G);

    if (warp >= kDecCW) {
        // ----------------------------------------------------------- producers
        // One lane of the first producer warp fills ring A with this CTA's
        // phase-1 items, one lane of the second ring B with its phase-2 items,
        // each as fast as slots free up (separate warps: neither spin-wait can
        // hold the other back).
        if (lane == 0) {
            const bool A = warp == kDecCW;
            const int n = A ? b1 - a1 : b2 - a2, N = A ? N1 : N2, S = A ? S1 : S2;
            uint8_t *ring = A ? ringA : ringB;
            uint64_t *fb = A ? full : full + N1, *eb = A ? empty : empty + N1;
            int k = 0;
            for (; k < n; k++) {
                const int slot = k % N;
                if (k >= N && !mbar_wait(&eb[slot], ((k / N) - 1) & 1, abort, p.status, 120, kDecWaitNs))
                    break;
                uint8_t *dst = ring + (size_t)slot * S;
                mbar_arrive_expect_tx(&fb[slot], S);
                if (A) {
                    const int gi = a1 + k, u = gi / per1, m0 = (gi - u * per1) * 8;
                    const size_t row = (size_t)R.uniq[u] * I + m0;
                    bulk_g2s(dst, p.gate_codes + row * (H / 2), 4 * H, &fb[slot]);
                    bulk_g2s(dst + 4 * H, p.up_codes + row * (H / 2), 4 * H, &fb[slot]);
                    bulk_g2s(dst + 8 * H, p.gate_scales + row * (H / 16), H / 2, &fb[slot]);
                    bulk_g2s(dst + 8 * H + H / 2, p.up_scales + row * (H / 16), H / 2, &fb[slot]);
                } else {
                    const int gi = a2 + k, u = gi / per2, r0 = (gi - u * per2) * 16;
                    const size_t row = (size_t)R.uniq[u] * H + r0;
                    bulk_g2s(dst, p.down_codes + row * (I / 2), 8 * I, &fb[slot]);
                    bulk_g2s(dst + 8 * I, p.down_scales + row * (I / 16), I, &fb[slot]);
                }
            }
            // The last fill of every slot must have landed before the CTA exits
            // (the consumers normally waited for each; not after an abort).
            for (int j = k - 1; j >= 0 && j >= k - N; j--)
                mbar_wait_drain(&fb[j % N], (j / N) & 1, kDecDrainNs);
        }
    } else {
        // ------------------------------------------------------ consumers
        // Per-token activation amax (this warp's rounds; every K round is covered
        // by every group), then the F16 B fragments.
        const bool int8 = p.act_type == NVFP4_MOE_ACT_INT8;
        if (!int8) {
            float m = 0.0f;
#pragma unroll
            for (int kk = 0; kk < kMaxRW; kk++) m = fmaxf(m, raw_amax(bx[kk]));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if (q == 0 && gq < T) atomicMax(&R.amax[gq], __float_as_uint(m));
        }
        named_bar(kBarConsumers, kDecCW * 32);
        if (threadIdx.x == 0) DEC_MARK(2);
        {
            const int sh = (int8 || gq >= T) ? 0 : pow2_shift_for(__uint_as_float(R.amax[gq]));
#pragma unroll
            for (int kk = 0; kk < kMaxRW; kk++) to_f16_frags(int8, sh, bx[kk]);
        }

        // ------------------------------------------- phase 1: gate/up + SwiGLU
        // A group of WG1 warps takes every groups1-th item of the CTA's range.
        // Each item's partial sums are reduced one iteration later by one warp of
        // the group (rotating), so that work overlaps the next item's MMAs.
        {
            const int groups1 = kDecCW / WG1, n1c = b1 - a1, w0 = g1 * WG1;
            const int nmine = n1c > g1 ? cdiv(n1c - g1, groups1) : 0;
            for (int it = 0; it <= nmine; it++) {
                const int k = g1 + it * groups1;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                if (it < nmine) {
                    const int slot = k % N1;
                    const bool got = warp_wait(&full[slot], (k / N1) & 1, abort, p.status, 121);
                    if (threadIdx.x == 0 && it == 0) DEC_MARK(3);
                    if (got) {
                        const uint8_t *base = ringA + (size_t)slot * S1;
#pragma unroll
                        for (int kk = 0; kk < kMaxRW; kk++) {
                            const int r = wi1 + kk * WG1;
                            if (r < NR1) {
                                uint4 ca, cb;
                                uint32_t sa, sb;
                                // rows 0..7 of the slot are gate rows, 8..15 the matching up rows
                                slot_round(base, H / 2, gq, gq + 8, r, q, ca, cb, sa, sb);
                                round_mma(acc, ca, cb, sa, sb, bx[kk]);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[slot]);
                }
                if (it > 0 && wi1 == (it - 1) % WG1) {
                    // item it - 1: the lane holds gate (x, y) and up (z, w) of
                    // intermediate m0 + gq for tokens 2q, 2q + 1
                    const float4 s = group_sum(part, w0, WG1, (it - 1) & 1, lane);
                    const int gi = a1 + k - groups1, u = gi / per1, m0 = (gi - u * per1) * 8;
                    const int e = R.uniq[u];
                    const float sg = __ldg(p.gate_global + e), su = __ldg(p.up_global + e);
                    bool fin = true;
#pragma unroll
                    for (int cc = 0; cc < 2; cc++) {
                        const int tok = 2 * q + cc;
                        const int pos = tok < T ? R.upos[u * kSlots + tok] : -1;
                        if (pos >= 0) {
                            const float xs = token_xscale(p, R, tok);
                            const float gv = (cc ? s.y : s.x) * sg * xs, uv = (cc ? s.w : s.z) * su * xs;
                            const float hf = silu(gv) * uv * exp2i(token_hexp(p, R, tok));
                            fin &= fits_f16(hf);
                            p.h[(size_t)pos * I + m0 + gq] = __float2half_rn(hf);
                        }
                    }
                    if (!fin) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfH | e);
                    __syncwarp();
                    if (lane == 0) red_release_add(ds + kDsReady + u, 1);
                }
                if (it < nmine)
                    part[((size_t)warp * 2 + (it & 1)) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                named_bar(1 + g1, WG1 * 32);
            }
        }

        // ------------------------------------------------ phase 2: down rows
        named_bar(kBarConsumers, kDecCW * 32);   // named barrier ids are reused below
        if (threadIdx.x == 0) DEC_MARK(4);
        {
            const int wi2 = warp % WG2, g2 = warp / WG2, w0 = g2 * WG2;
            const int groups2 = kDecCW / WG2, n2c = b2 - a2;
            const int nmine = n2c > g2 ? cdiv(n2c - g2, groups2) : 0;
            int cur_u = -1;
            for (int it = 0; it <= nmine; it++) {
                const int k = g2 + it * groups2;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                if (it < nmine) {
                    const int gi = a2 + k, u = gi / per2;
                    if (u != cur_u) {
                        // this expert's h rows, once all its phase-1 items are done
                        int ok = 1;
                        if (lane == 0) ok = wait_geq(ds + kDsReady + u, per1, p.status, 102);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) *abort = 1;
                        const int pos = gq < T ? R.upos[u * kSlots + gq] : -1;
#pragma unroll
                        for (int kk = 0; kk < kMaxRW; kk++) {
                            const int k0 = 128 * (wi2 + kk * WG2) + 32 * q;
                            if (pos >= 0 && k0 < I) {
                                const uint4 *s = reinterpret_cast<const uint4 *>(p.h + (size_t)pos * I + k0);
#pragma unroll
                                for (int i = 0; i < 4; i++) bx[kk][i] = __ldcg(s + i);
                            } else {
#pragma unroll
                                for (int i = 0; i < 4; i++) bx[kk][i] = make_uint4(0, 0, 0, 0);
                            }
                        }
                        cur_u = u;
                        if (threadIdx.x == 0 && it == 0) DEC_MARK(5);
                    }
                    const int slot = k % N2;
                    if (warp_wait(&full[N1 + slot], (k / N2) & 1, abort, p.status, 122)) {
                        const uint8_t *base = ringB + (size_t)slot * S2;
#pragma unroll
                        for (int kk = 0; kk < kMaxRW; kk++) {
                            const int r = wi2 + kk * WG2;
                            if (r < NR2) {
                                uint4 ca, cb;
                                uint32_t sa, sb;
                                slot_round(base, I / 2, gq, gq + 8, r, q, ca, cb, sa, sb);
                                round_mma(acc, ca, cb, sa, sb, bx[kk]);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[N1 + slot]);
                }
                if (it > 0 && wi2 == (it - 1) % WG2) {
                    // item it - 1: w * s_d * y of hidden rows r0 + gq (x, y) and
                    // r0 + gq + 8 (z, w), tokens 2q and 2q + 1, into the pairs' FP32
                    // rows (h was stored times 2^hexp; undone here)
                    const float4 s = group_sum(part, w0, WG2, (it - 1) & 1, lane);
                    const int gi = a2 + k - groups2, u = gi / per2, r0 = (gi - u * per2) * 16;
                    const int e = R.uniq[u];
                    const float sd = __ldg(p.down_global + e);
                    bool fin = true;
#pragma unroll
                    for (int cc = 0; cc < 2; cc++) {
                        const int tok = 2 * q + cc;
                        const int pos = tok < T ? R.upos[u * kSlots + tok] : -1;
                        if (pos >= 0) {
                            const float w = R.uw[u * kSlots + tok] * sd * exp2i(-token_hexp(p, R, tok));
                            const float y0 = (cc ? s.y : s.x) * w, y1 = (cc ? s.w : s.z) * w;
                            fin &= isfinite(y0) && isfinite(y1);
                            p.ybuf[(size_t)pos * H + r0 + gq] = y0;
                            p.ybuf[(size_t)pos * H + r0 + gq + 8] = y1;
                        }
                    }
                    if (!fin) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfY | e);
                }
                if (it < nmine)
                    part[((size_t)warp * 2 + (it & 1)) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                named_bar(1 + g2, WG2 * 32);
            }
        }

        // ------------------------------------------ weighted combine into out
        // Once every CTA's down rows are written (which also means every CTA has
        // read the activations, which out may alias), each CTA adds up its share
        // of the hidden rows: out_t (+)= sum_j rows(t, j), in order j = 0..K-1.
        named_bar(kBarConsumers, kDecCW * 32);
        if (threadIdx.x == 0) {
            if (!((p.test_flags & NVFP4_MOE_TEST_DECODE_STALL) && blockIdx.x == 0))
                red_release_add(ds + kDsDone, 1);
            DEC_MARK(5 + 1);
            s_ok = wait_geq(ds + kDsDone, G, p.status, 101);
        }
        named_bar(kBarConsumers, kDecCW * 32);
        if (s_ok) {
            const int rlo = (int)((long long)H * c / G), rhi = (int)((long long)H * (c + 1) / G);
            const int nrow = rhi - rlo;
            bool fo = true;
            for (int o = threadIdx.x; o < nrow * T; o += kDecCW * 32) {
                const int t = o / nrow, row = rlo + (o - t * nrow);
                float y[NVFP4_MOE_MAX_TOPK];
#pragma unroll
                for (int j = 0; j < NVFP4_MOE_MAX_TOPK; j++)
                    y[j] = j < K ? __ldcg(p.ybuf + (size_t)R.pos[t * K + j] * H + row) : 0.0f;
                float sum = 0.0f;
#pragma unroll
                for (int j = 0; j < NVFP4_MOE_MAX_TOPK; j++)
                    if (j < K) sum += y[j];
                float *op = p.out + (size_t)t * H + row;
                const float v = p.out_add ? *op + sum : sum;
                fo &= isfinite(v);
                *op = v;
            }
            if (!fo) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfOut | rlo);
        }
    }

    __syncthreads();
    if (blockIdx.x == 0) publish_route(p, R);
    // The last CTA done resets the counters for the next launch.
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(ds + kDsExit, 1) == G - 1) {
            for (int u = 0; u < U; u++) ds[kDsReady + u] = 0;
            ds[kDsDone] = 0;
            ds[kDsExit] = 0;
            __threadfence();
        }
        DEC_MARK(7);
    }
    // The next layer's grid may launch once every CTA is here.
    grid_dep_launch();
}

#ifdef NVMOE_DEC_TRACE
}  // namespace nvmoe
extern "C" NVFP4_MOE_API int nvfp4_moe_dbg_trace(unsigned long long *host, int n) {
    return (int)cudaMemcpyFromSymbol(host, nvmoe::g_dec_trace, sizeof(unsigned long long) * n);
}
namespace nvmoe {
#endif

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

int decode_grid() { return sm_count(); }

// Ring slots: about half the budget for phase-1 items (at most 8), the rest for
// phase-2 items (at most 32).
static void decode_plan(int H, int I, int &n1, int &n2) {
    const int avail = kDecSmemBudget - kPartBytes - 16 * (8 + 32);   // barriers at most
    const int s1 = 9 * H, s2 = 9 * I;
    n1 = min(8, max(2, avail / 2 / s1));
    n2 = min(32, (avail - n1 * s1) / s2);
}

bool decode_fits(int H, int I) {
    if (H % 32 || I % 32) return false;
    if (dec_group_warps(cdiv(H, 128)) == 0 || dec_group_warps(cdiv(I, 128)) == 0) return false;
    int n1, n2;
    decode_plan(H, I, n1, n2);
    return n2 >= 2 && 2 * 9 * H <= kDecSmemBudget - kPartBytes;
}

static size_t decode_smem(int H, int I, int n1, int n2) {
    return (size_t)kPartBytes + (size_t)n1 * 9 * H + (size_t)n2 * 9 * I + 16 * (size_t)(n1 + n2);
}

template <int NPER>
static cudaError_t launch_layer(Params p, cudaStream_t s) {
    decode_plan(p.H, p.I, p.dec_n1, p.dec_n2);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(decode_grid());
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = decode_smem(p.H, p.I, p.dec_n1, p.dec_n2);
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
    // dynamic shared memory above the 48 KB default: the rings take most of the SM
    const int big = kDecSmemBudget;
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
