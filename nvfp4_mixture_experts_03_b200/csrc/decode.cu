// Decode path (T <= 8): stream each selected expert's 4.5-bit weights once.
//
// The pages keep the quality profile on "canonical FP32 expert decode" ("#1858
// ... strata-safetensors", "What do you want to do?" and the paragraph after
// the measurements) and note that a decode round is bound by moving expert
// bytes ("Strata NVFP4" README, "Limits"). On B200 every expert is resident in
// HBM, so decode is a pure HBM stream whose time is set by how early the weight
// loads start, how many are in flight, and how few round trips lie between them.
//
// One kernel per layer, one 16-warp CTA per SM, launched with programmatic
// dependent launch:
//   routing: every CTA routes the <= 8 tokens itself (warp top-k per token, then
//     positions by counting), and stages the activations as F16 in shared
//     memory (its first weight loads are already in flight by then);
//   gate/up + SwiGLU: the flattened space of (used expert, 8 intermediates)
//     granules is cut into equal contiguous ranges, one per CTA; a CTA splits
//     its (granule, 128-wide K round) units evenly over its warps, sums a granule
//     split between warps in shared memory in warp order, and stores h (F16 with
//     a per-token power-of-two range exponent) at each pair's position;
//   one grid barrier (bounded wait; the last CTA to arrive resets the count and
//     bumps a generation word the others wait on): every h is stored, every CTA has read the
//     activations (out may alias them);
//   down + weighted combine: each CTA owns whole 16-row blocks of out and, for
//     every used expert, streams those rows of the expert's down matrix (whole
//     rows: contiguous bytes, which DRAM serves about twice as fast as a column
//     slice of the same size), with every pair's h row staged in shared memory.
//     Per row block the experts are summed in registers in ascending order
//     (scaled by w * s_d), a block split between warps in warp order, and the
//     rows of out are stored once, in FP32.
// Determinism: every sum runs in a fixed order and no value is added by an
// atomic, so the result is the same bits on every run.
// Arithmetic: each weight is decoded exactly to F16 (E2M1 -> F16 conversion
// times its E4M3 group scale: at most 6 significant bits, exact in F16) and fed
// to mma.sync m16n8k16 with the token slots as N, FP32 accumulation; the tensor
// scale and the per-token activation scale are applied to the FP32 result.
//
// Fragment mapping (m16n8k16, A row-major, B col-major): thread (g = lane/4,
// q = lane%4) holds rows g and g+8. It loads 16 contiguous code bytes of each
// row per 128-wide K round (byte offset 64*r + 16*q), so a warp reads whole
// 32-byte sectors. Mma step s of round r uses physical K 128r + 32q + 4s +
// {0,1,2,3} for logical K {2q, 2q+1, 2q+8, 2q+9}; the activations and h use the
// same permutation, so every dot product is the plain one. H and I need only be
// multiples of 32: a 32-wide piece of a round past the end is zero on both sides.
#include "common.cuh"
#include "route_common.cuh"
#include "stream_common.cuh"

namespace nvmoe {


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

constexpr int kDecWarps = kDecWarpsPerCta;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kGuRounds = 4;   // gate/up: 128-wide K rounds of loads one warp holds per chunk
constexpr int kDnUnits = 3;    // down: (16 rows, expert, 128-wide K round) units one warp holds per chunk
constexpr int kMaxPairs = NVFP4_MOE_DECODE_MAX_T * NVFP4_MOE_MAX_TOPK;  // 128
constexpr int kSlots = NVFP4_MOE_DECODE_MAX_T;

constexpr uint64_t kDecWaitNs = 200000000ull;   // grid barrier wait limit (200 ms)

// The weight planes and router logits of the layer being run (in shared memory:
// a stack of layers swaps them per layer, the parameters stay constant).
struct DecLayer {
    const uint8_t *gate_codes, *up_codes, *gate_scales, *up_scales;
    const float *gate_global, *up_global;
    const uint8_t *down_codes, *down_scales;
    const float *down_global;
    const float *logits;
};

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
    float dw[kMaxPairs * kSlots];   // w * s_d * 2^-hexp of (used expert, token), 0 if absent
    unsigned amax[kSlots];          // per-token activation amax (FP32 bits)
    float xsc[kSlots];              // per-token factor that undoes the F16 staging scale
    int hexp[kSlots];               // per-token exponent h is stored with (h_exp_for)
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
// shared scratch each. Warps kSlots.. (which route no token) run `side` meanwhile.
template <int NPER, class Side>
__device__ void cta_route(const Params &p, const float *logits, DecRoute &R, bool report, int *ex, int *sc,
                          Side side) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.T * p.K, E = p.E;
    for (int i = threadIdx.x; i < kMaxPairs * kSlots; i += blockDim.x) R.upos[i] = -1;
    for (int i = threadIdx.x; i < E; i += blockDim.x) ex[i] = 0;
    if (threadIdx.x < kSlots) R.amax[threadIdx.x] = 0u;
    __syncthreads();
    if (warp < p.T) {
        int id;
        float w;
        if (logits) {
            bool finite;
            warp_topk<NPER>(logits + (size_t)warp * E, E, p.K, lane, id, w, finite);
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
    } else if (warp >= kSlots) {
        side();
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
        if (within == 0) {
            R.uniq[u] = e;
            R.uoff[u] = rank;
        }
    }
    if (threadIdx.x == 0) {
        R.U = total >> 16;
        R.uoff[total >> 16] = P;
    }
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

// A CTA's share of the gate/up phase: granules [gb, ge) of the flattened (used
// expert, 8 intermediates) space.
struct DecPlan {
    int gb, ge;
    int ok;     // the grid barrier completed
    int last;   // this CTA finished last (resets the counters)
};

constexpr int kMaxStackLayers = NVFP4_MOE_MAX_STACK;
struct DecStack {
    int32_t n;
    const float *logits;   // [n][T][E]
    DecLayer layer[kMaxStackLayers];
};

// Gate/up weights of one warp's chunk: rows g (gate) and g+8 (up), up to
// kGuRounds rounds. Scales: per round, row g's two scale bytes in bits 0..15 of
// s[j] and row g+8's in 16..31; or, when whole 8-byte scale pieces can be read
// (gu_issue's `vec`), round r0 + q's eight bytes of row g in s[0..1] and of row
// g+8 in s[2..3], which gu_scales hands to the four lanes of the quad.
struct GuBuf {
    uint4 ca[kGuRounds], cb[kGuRounds];
    uint32_t s[kGuRounds];
};
static_assert(kGuRounds == 4, "a quad's four lanes fetch the scale pieces of a chunk's four rounds");

// A run of at most kGuRounds consecutive K rounds of one granule (CTA-local).
struct Chunk {
    int item, r0, r1;   // r1 == 0: none
};

// Next chunk of the unit range [x, end) (units = item * R + round); advances x.
__device__ inline Chunk take_chunk(int &x, int end, int R) {
    Chunk c{0, 0, 0};
    if (x < end) {
        c.item = x / R;
        c.r0 = x - c.item * R;
        c.r1 = min(min(R, c.r0 + kGuRounds), end - c.item * R);
        x = c.item * R + c.r1;
    }
    return c;
}

// Weight loads of rounds [c.r0, c.r1) of granule P.gb + c.item; 16-byte pieces
// past the row's end (H not a multiple of 128) are zero, with zero scales.
// `vec` (H a multiple of 128, 8-byte aligned scale planes): lane q of the quad
// fetches round c.r0 + q's eight scale bytes of both rows in one load each,
// instead of every lane fetching two bytes of every round.
__device__ inline void gu_issue(const Params &p, const DecLayer &W, const DecRoute &R, const DecPlan &P,
                                const Chunk &c, int g, int q, bool vec, GuBuf &b) {
    if (c.r1 == 0) return;
    const int per_u = p.I / 8, gi = P.gb + c.item, u = gi / per_u;
    const size_t ra = (size_t)R.uniq[u] * p.I + (gi - u * per_u) * 8 + g;
    const int kb = p.H / 2;
    const uint8_t *ca_p = W.gate_codes + ra * kb, *cb_p = W.up_codes + ra * kb;
    const uint8_t *sa_p = W.gate_scales + ra * (p.H / 16), *sb_p = W.up_scales + ra * (p.H / 16);
    if (vec) {
        // Every piece lies inside its row, so every load is unconditional (rounds
        // past c.r1 repeat round c.r1 - 1, unused): each lands straight in its
        // buffer register, with no select that would wait for it here.
        const int rq = min(c.r0 + q, c.r1 - 1);
        const uint2 va = __ldg(reinterpret_cast<const uint2 *>(sa_p + 8 * rq));
        const uint2 vb = __ldg(reinterpret_cast<const uint2 *>(sb_p + 8 * rq));
        b.s[0] = va.x;
        b.s[1] = va.y;
        b.s[2] = vb.x;
        b.s[3] = vb.y;
#pragma unroll
        for (int j = 0; j < kGuRounds; j++) {
            const int r = min(c.r0 + j, c.r1 - 1);
            b.ca[j] = ldg_stream(ca_p + 64 * r + 16 * q);
            b.cb[j] = ldg_stream(cb_p + 64 * r + 16 * q);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < kGuRounds; j++) {
        const int r = c.r0 + j;
        if (r < c.r1) {
            if (64 * r + 16 * q < kb) {
                b.ca[j] = ldg_stream(ca_p + 64 * r + 16 * q);
                b.cb[j] = ldg_stream(cb_p + 64 * r + 16 * q);
                b.s[j] = (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(sa_p + 8 * r + 2 * q)) |
                         ((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(sb_p + 8 * r + 2 * q)) << 16);
            } else {
                b.ca[j] = b.cb[j] = make_uint4(0, 0, 0, 0);
                b.s[j] = 0;
            }
        }
    }
}

// Round j's scale bytes of this lane (row g in bits 0..15, row g+8 in 16..31)
// from a chunk loaded with gu_issue's `vec`: lane j of the quad holds round
// r0 + j's eight bytes of each row; this lane (q) takes bytes 2q and 2q + 1.
// Every lane of the warp calls it (shuffles).
__device__ inline uint32_t gu_scales(const GuBuf &b, int j, int lane, int q) {
    const int src = (lane & ~3) | j;
    const uint32_t a0 = __shfl_sync(0xffffffffu, b.s[0], src), a1 = __shfl_sync(0xffffffffu, b.s[1], src);
    const uint32_t b0 = __shfl_sync(0xffffffffu, b.s[2], src), b1 = __shfl_sync(0xffffffffu, b.s[3], src);
    const int sh = 16 * (q & 1);
    const uint32_t sa = ((q >> 1) ? a1 : a0) >> sh, sb = ((q >> 1) ? b1 : b0) >> sh;
    return (sa & 0xFFFFu) | (sb << 16);
}

// h of granule P.gb + j for this thread's intermediate (row g) and token slots
// 2q, 2q+1 whose token chose the expert, from the granule's full sums (gate: v.x,
// v.y; up: v.z, v.w), stored F16 at the pair's position.
__device__ inline void swiglu_store(const Params &p, const DecRoute &R, const DecPlan &P,
                                    const float *gsc, int j, float4 v, int g, int q, int &bad) {
    const int per_u = p.I / 8, gi = P.gb + j, u = gi / per_u, e = R.uniq[u];
    const int i = (gi - u * per_u) * 8 + g;
    const float sg = gsc[e], su = gsc[p.E + e];
    const float gs[2] = {v.x, v.y}, us[2] = {v.z, v.w};
#pragma unroll
    for (int c = 0; c < 2; c++) {
        const int slot = 2 * q + c;
        const int pos = slot < p.T ? R.upos[u * kSlots + slot] : -1;
        if (pos >= 0) {
            const float gv = gs[c] * sg * R.xsc[slot], uv = us[c] * su * R.xsc[slot];
            const float hf = silu(gv) * uv * exp2i(R.hexp[slot]);
            if (!fits_f16(hf)) bad = e;
            p.h[(size_t)pos * p.I + i] = __float2half_rn(hf);
        }
    }
}

// Down weights of one warp's chunk: kDnUnits units (16-row block, used expert,
// 128-wide K round), rows g and g+8, 16 code bytes and two scale bytes each.
// The two scale bytes of each row stay in their own registers as loaded: a
// combining instruction at issue time would wait there for the loads to land.
struct DnBuf {
    uint4 ca[kDnUnits], cb[kDnUnits];
    uint32_t sa[kDnUnits], sb[kDnUnits];   // rows g and g+8: two scale bytes each
};

// Position of a down unit of the CTA (row blocks rb0.., U experts, R2 rounds
// each): row block (CTA-local), used expert, round; stepped without division.
struct DnCur {
    int rbl, u, r;
};
__device__ inline DnCur dn_cur(int x, int U, int R2) {
    DnCur c;
    const int per_rb = U * R2;
    c.rbl = x / per_rb;
    const int rem = x - c.rbl * per_rb;
    c.u = rem / R2;
    c.r = rem - c.u * R2;
    return c;
}
__device__ inline void dn_next(DnCur &c, int U, int R2) {
    if (++c.r == R2) {
        c.r = 0;
        if (++c.u == U) {
            c.u = 0;
            c.rbl++;
        }
    }
}

// Loads of the n <= kDnUnits down units from c on; 16-byte pieces past the row's
// end (I not a multiple of 128) are zero, with zero scales.
__device__ inline void dn_issue(const Params &p, const DecLayer &W, const DecRoute &R, int rb0, DnCur c,
                                int n, int g, int q, bool full, DnBuf &b) {
    const int H = p.H, I = p.I, R2 = cdiv(I, 128), U = R.U;
    if (full) {
        if (n <= 0) return;
        // I a multiple of 128: every piece lies inside its row and every load is
        // unconditional (units past n repeat unit n - 1, unused), landing straight
        // in its buffer register
#pragma unroll
        for (int j = 0; j < kDnUnits; j++) {
            const size_t ra = (size_t)R.uniq[c.u] * H + 16 * (rb0 + c.rbl) + g;
            const uint8_t *cp = W.down_codes + ra * (I / 2) + 64 * c.r + 16 * q;
            const uint8_t *sp = W.down_scales + ra * (I / 16) + 8 * c.r + 2 * q;
            b.ca[j] = ldg_stream(cp);
            b.cb[j] = ldg_stream(cp + 8 * (I / 2));
            b.sa[j] = __ldg(reinterpret_cast<const unsigned short *>(sp));
            b.sb[j] = __ldg(reinterpret_cast<const unsigned short *>(sp + 8 * (I / 16)));
            if (j + 1 < n) dn_next(c, U, R2);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < kDnUnits; j++) {
        if (j < n) {
            if (64 * c.r + 16 * q < I / 2) {
                const size_t ra = (size_t)R.uniq[c.u] * H + 16 * (rb0 + c.rbl) + g;
                const uint8_t *cp = W.down_codes + ra * (I / 2) + 64 * c.r + 16 * q;
                const uint8_t *sp = W.down_scales + ra * (I / 16) + 8 * c.r + 2 * q;
                b.ca[j] = ldg_stream(cp);
                b.cb[j] = ldg_stream(cp + 8 * (I / 2));
                b.sa[j] = __ldg(reinterpret_cast<const unsigned short *>(sp));
                b.sb[j] = __ldg(reinterpret_cast<const unsigned short *>(sp + 8 * (I / 16)));
            } else {
                b.ca[j] = b.cb[j] = make_uint4(0, 0, 0, 0);
                b.sa[j] = b.sb[j] = 0;
            }
            dn_next(c, U, R2);
        }
    }
}

// out rows 16 rb + g and + 8, token slots 2q, 2q+1 < T, from this thread's sums.
__device__ inline void store_out(const Params &p, int rb, const float4 &v, int g, int q, int &bad) {
    const float f[4] = {v.x, v.y, v.z, v.w};   // (row g: slots 2q, 2q+1), (row g+8: same)
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const int slot = 2 * q + (k & 1), row = 16 * rb + g + 8 * (k >> 1);
        if (slot < p.T) {
            const size_t o = (size_t)slot * p.H + row;
            const float r = p.out_add ? p.out[o] + f[k] : f[k];
            if (!isfinite(r)) bad = row;
            p.out[o] = r;
        }
    }
}

// Bounded wait until *word != old (one thread); latches TIMEOUT on give-up.
__device__ inline bool wait_ne(const int32_t *word, int old, int32_t *status, int where) {
    const volatile int32_t *v = word;
    if (*v != old) return true;
    const uint64_t t0 = globaltimer();
    while (*v == old) {
        __nanosleep(32);
        if (globaltimer() - t0 > kDecWaitNs) {
            latch_status(status, NVFP4_MOE_ERR_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

// Row strides (F16 elements) of the activation tile and of the staged h rows:
// the K rounds rounded up, plus a few elements so that rows fall in different
// banks.
__host__ __device__ inline int dec_ld1(int H) { return cdiv(H, 128) * 128 + 4; }
// Bytes of the activation tile, rounded up to 16 (the parts after it are float4).
__host__ __device__ inline size_t dec_xs_bytes(int T, int H) {
    return ((size_t)(T + 1) * dec_ld1(H) * 2 + 15) & ~(size_t)15;
}
__host__ __device__ inline int dec_ld2(int I) { return cdiv(I, 128) * 128 + 8; }

// The warp (of W) whose share of n units holds unit x.
__device__ inline int owner(int n, int W, int x) {
    int w = (int)(((long long)x * W) / n);   // close; fix up against the exact shares
    int a, b;
    share(n, w, W, a, b);
    while (x < a) share(n, --w, W, a, b);
    while (x >= b) share(n, ++w, W, a, b);
    return w;
}

// Generation-counting grid barrier: thread 0 of every CTA arrives; the last to
// arrive resets the count and bumps the generation word the others wait on
// (bounded). `gen` (thread 0's copy) is the generation being waited out; it
// advances with each barrier. Returns, in every thread, whether it completed.
__device__ inline bool grid_barrier(const Params &p, int32_t *ds, int &gen, int where, bool arrive,
                                    int *ok_smem) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        bool open = false;
        if (arrive && atomicAdd(ds + kDsArrive, 1) == (int)gridDim.x - 1) {
            atomicExch(ds + kDsArrive, 0);
            __threadfence();
            atomicAdd(ds + kDsGen, 1);
            open = true;
        }
        *ok_smem = open || wait_ne(ds + kDsGen, gen, p.status, where);
        gen++;
        __threadfence();
    }
    __syncthreads();
    return *ok_smem != 0;
}

// One decode layer (routing, gate/up + SwiGLU, grid barrier, down + combine).
template <int NPER>
__device__ __forceinline__ void decode_body(const Params &p, const DecLayer &W, DecRoute &R, DecPlan &P,
                                            uint8_t *dsm, int &gen) {
    const int H = p.H, I = p.I, T = p.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int ld1 = dec_ld1(H), ld2 = dec_ld2(I);
    // gate/up phase: [T + 1][ld1] F16 activations (row T: zeros, for the token
    // slots past T), split-granule parts;
    // down phase (same storage): [P + 1][ld2] h rows (row P: zeros), split-row-block parts
    __half *xs = reinterpret_cast<__half *>(dsm);
    float4 *part1 = reinterpret_cast<float4 *>(dsm + dec_xs_bytes(T, H));   // 16-byte aligned
    __half *hs = reinterpret_cast<__half *>(dsm);
    float4 *part2 = reinterpret_cast<float4 *>(hs + (size_t)(p.T * p.K + 1) * ld2);
    int *scratch = reinterpret_cast<int *>(dsm + p.dec_union);   // routing: 2E ints
    float *gsc = reinterpret_cast<float *>(scratch + 2 * p.E);    // [gate, up, down][E] global scales
    int32_t *ds = p.dstate;

    // While warps 0..T-1 route, warps 8..15 stage the activations: per-token amax
    // -> power-of-two shift -> F16 in shared memory (columns past H and the zero
    // row T are zero), and fetch every expert's three global scales.
    const bool int8 = p.act_type == NVFP4_MOE_ACT_INT8;
    auto stage = [&]() {
        const int st = threadIdx.x - kSlots * 32, sw = st >> 5, nst = kDecThreads - kSlots * 32;
        for (int e = st; e < p.E; e += nst) {
            gsc[e] = W.gate_global[e];
            gsc[p.E + e] = W.up_global[e];
            gsc[2 * p.E + e] = W.down_global[e];
        }
        const int h8 = H / 8, p8 = ld1 / 8;
        for (int c = st; c < T * (p8 - h8) + p8; c += nst) {
            int t, k8;
            if (c < T * (p8 - h8)) { t = c / (p8 - h8); k8 = h8 + c % (p8 - h8); }
            else { t = T; k8 = c - T * (p8 - h8); }
            uint2 *dst = reinterpret_cast<uint2 *>(xs + (size_t)t * ld1 + 8 * k8);
            dst[0] = make_uint2(0, 0);
            if (8 * k8 + 4 < ld1) dst[1] = make_uint2(0, 0);
        }
        if (!int8) {
            for (int t = sw; t < T; t += nst / 32) {
                float m = 0.0f;
                for (int k8 = lane; k8 < h8; k8 += 32) {
                    float v[8];
                    load_act8(p, t, k8, v);
#pragma unroll
                    for (int j = 0; j < 8; j++) m = fmaxf(m, fabsf(v[j]));
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) R.amax[t] = __float_as_uint(m);
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(nst) : "memory");
        for (int c = st; c < T * h8; c += nst) {
            const int t = c / h8, k8 = c - t * h8;
            const int sh = int8 ? 0 : pow2_shift_for(__uint_as_float(R.amax[t]));
            float v[8];
            load_act8(p, t, k8, v);
            const uint4 pk = pack8_f16(v, sh);
            uint2 *dst = reinterpret_cast<uint2 *>(xs + (size_t)t * ld1 + 8 * k8);
            dst[0] = make_uint2(pk.x, pk.y);
            dst[1] = make_uint2(pk.z, pk.w);
        }
        if (st < T) {
            const float am = int8 ? 127.0f * p.act_scale[st] : __uint_as_float(R.amax[st]);
            R.xsc[st] = int8 ? p.act_scale[st] : exp2i(-pow2_shift_for(am));
            R.hexp[st] = h_exp_for(am);
        }
    };
    cta_route<NPER>(p, W.logits, R, blockIdx.x == 0, scratch, scratch + p.E, stage);
    const int U = R.U;
    const int n8 = U * (I / 8);
    const int gb = (int)((long long)n8 * blockIdx.x / gridDim.x);
    const int ge = (int)((long long)n8 * (blockIdx.x + 1) / gridDim.x);
    if (threadIdx.x == 0) {
        P.gb = gb;
        P.ge = ge;
    }

    // this warp's gate/up share; its first loads go out before the activations
    // are staged
    const int R1 = cdiv(H, 128), R2 = cdiv(I, 128);
    const bool gvec = H % 128 == 0 && ((uintptr_t)W.gate_scales | (uintptr_t)W.up_scales) % 8 == 0;
    const bool dfull = I % 128 == 0;
    const int n1 = (ge - gb) * R1;
    int a1, b1;
    share(n1, warp, kDecWarps, a1, b1);
    int x1 = a1;
    Chunk cur = take_chunk(x1, b1, R1);
    GuBuf buf0, buf1;
    {
        const DecPlan Pl{gb, ge, 0, 0};
        gu_issue(p, W, R, Pl, cur, g, q, gvec, buf0);
    }

    __syncthreads();   // P is read by every warp from here on

    // gate/up + SwiGLU: a granule whole in this warp goes to h from registers; a
    // split one leaves its part in part1 (slot 0: the warp's first granule,
    // slot 1: its last)
    int bad1 = -1;   // expert of a non-finite value this thread saw
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        int seg_r0 = cur.r0;
        const int first_item = a1 / R1;
        const __half *xrow = xs + (size_t)(g < T ? g : T) * ld1 + 32 * q;
        auto step = [&](GuBuf &b, GuBuf &nb) {
            const Chunk nxt = take_chunk(x1, b1, R1);
            gu_issue(p, W, R, P, nxt, g, q, gvec, nb);
#pragma unroll
            for (int j = 0; j < kGuRounds; j++) {
                const int r = cur.r0 + j;
                if (r < cur.r1) {
                    const __half *xr = xrow + 128 * r;
                    const uint32_t sj = gvec ? gu_scales(b, j, lane, q) : b.s[j];
                    round_mma(acc, b.ca[j], b.cb[j], sj & 0xFFFF, sj >> 16,
                              [&](int s, uint32_t &v0, uint32_t &v1) {
                                  const uint2 v = *reinterpret_cast<const uint2 *>(xr + 4 * s);
                                  v0 = v.x;
                                  v1 = v.y;
                              });
                }
            }
            if (nxt.r1 == 0 || nxt.item != cur.item) {
                const float4 v = make_float4(acc[0], acc[1], acc[2], acc[3]);
                if (cur.r1 - seg_r0 == R1)
                    swiglu_store(p, R, P, gsc, cur.item, v, g, q, bad1);
                else
                    part1[(warp * 2 + (cur.item == first_item ? 0 : 1)) * 32 + lane] = v;
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

    // this CTA's down share: whole 16-row blocks of out, every used expert; the
    // warp's first loads go out before the barriers
    int rb0, rb1;
    share(H / 16, blockIdx.x, gridDim.x, rb0, rb1);
    const int n2 = (rb1 - rb0) * U * R2;
    int a2, b2;
    share(n2, warp, kDecWarps, a2, b2);
    DnBuf d0, d1;
    dn_issue(p, W, R, rb0, dn_cur(a2, U, R2), min(kDnUnits, b2 - a2), g, q, dfull, d0);
    __syncthreads();
    // granules split between warps: their parts summed in warp order
    for (int j = warp; j < ge - gb; j += kDecWarps) {
        const int w0 = owner(n1, kDecWarps, j * R1), w1 = owner(n1, kDecWarps, j * R1 + R1 - 1);
        if (w0 == w1) continue;   // whole in one warp: already stored
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = w0; w <= w1; w++) {
            int wa, wb;
            share(n1, w, kDecWarps, wa, wb);
            if (wa == wb) continue;
            const float4 v = part1[(w * 2 + (j == wa / R1 ? 0 : 1)) * 32 + lane];
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        swiglu_store(p, R, P, gsc, j, s, g, q, bad1);
    }
    warp_report(p, bad1, kNfH);
    // per (used expert, token slot): w * s_d * 2^-hexp (0 where the token did not
    // choose the expert)
    for (int k = threadIdx.x; k < U * kSlots; k += blockDim.x) {
        const int u = k / kSlots, slot = k - u * kSlots;
        const int pos = slot < T ? R.upos[k] : -1;
        R.dw[k] = pos >= 0 ? R.uw[k] * gsc[2 * p.E + R.uniq[u]] * exp2i(-R.hexp[slot]) : 0.0f;
    }

    // grid barrier: every CTA's h is stored (and every CTA has read the
    // activations: out may alias them)
    grid_barrier(p, ds, gen, 101, !((p.test_flags & NVFP4_MOE_TEST_DECODE_STALL) && blockIdx.x == 0),
                 &P.ok);
    if (P.ok && n2 > 0) {
        // every pair's h row, K past I zero, then a zero row for absent tokens
        const int per_row = ld2 / 8, P2 = T * p.K;   // 16-byte pieces per row; pairs
        for (int c = threadIdx.x; c < (P2 + 1) * per_row; c += blockDim.x) {
            const int r = c / per_row, k = c - r * per_row;
            __half *dst = hs + (size_t)r * ld2 + 8 * k;
            if (r < P2 && 8 * k < I) cp_async16(dst, p.h + (size_t)r * I + 8 * k);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
        }
        asm volatile("cp.async.commit_group;\n cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();

    // down + weighted combine, in registers: per (row block, expert) the K rounds
    // sum in acc, then oacc += acc * w * s_d; a row block whole in this warp is
    // stored from registers, a split one leaves its part in part2
    int bad2 = -1;
    if (P.ok) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, oacc[4] = {0.f, 0.f, 0.f, 0.f};
        const int first_rb = a2 / (U * R2);
        int seg0 = a2;   // first unit of the current row block's part in this warp
        int x = a2;
        DnCur cc = dn_cur(a2, U, R2);   // compute cursor: unit x
        auto step = [&](DnBuf &b, DnBuf &nb) {
            const int xn = x + kDnUnits;
            if (xn < b2) {
                DnCur ic = cc;   // the next chunk starts kDnUnits units on
#pragma unroll
                for (int j = 0; j < kDnUnits; j++) dn_next(ic, U, R2);
                dn_issue(p, W, R, rb0, ic, min(kDnUnits, b2 - xn), g, q, dfull, nb);
            }
#pragma unroll
            for (int j = 0; j < kDnUnits; j++) {
                const int xx = x + j;
                if (xx < b2) {
                    const int rbl = cc.rbl, u = cc.u, r = cc.r;
                    dn_next(cc, U, R2);
                    const int pos = g < T ? R.upos[u * kSlots + g] : -1;
                    const __half *hr = hs + (size_t)(pos >= 0 ? pos : T * p.K) * ld2 + 128 * r + 32 * q;
                    round_mma(acc, b.ca[j], b.cb[j], b.sa[j], b.sb[j],
                              [&](int s, uint32_t &v0, uint32_t &v1) {
                                  const uint2 v = *reinterpret_cast<const uint2 *>(hr + 4 * s);
                                  v0 = v.x;
                                  v1 = v.y;
                              });
                    const bool last_unit = xx + 1 == b2;
                    if (r == R2 - 1 || last_unit) {   // expert u done for this row block
                        const float w0 = R.dw[u * kSlots + 2 * q], w1 = R.dw[u * kSlots + 2 * q + 1];
                        oacc[0] += acc[0] * w0;
                        oacc[1] += acc[1] * w1;
                        oacc[2] += acc[2] * w0;
                        oacc[3] += acc[3] * w1;
#pragma unroll
                        for (int c = 0; c < 4; c++) acc[c] = 0.0f;
                        if (u == U - 1 || last_unit) {   // row block done in this warp
                            const float4 o4 = make_float4(oacc[0], oacc[1], oacc[2], oacc[3]);
                            const bool whole = seg0 == rbl * U * R2 && (r == R2 - 1 && u == U - 1);
                            if (whole)
                                store_out(p, rb0 + rbl, o4, g, q, bad2);
                            else
                                part2[(warp * 2 + (rbl == first_rb ? 0 : 1)) * 32 + lane] = o4;
#pragma unroll
                            for (int c = 0; c < 4; c++) oacc[c] = 0.0f;
                            seg0 = xx + 1;
                        }
                    }
                }
            }
            x = xn;
        };
        while (x < b2) {
            step(d0, d1);
            if (x >= b2) break;
            step(d1, d0);
        }
    }
    __syncthreads();
    // row blocks split between warps: their parts summed in warp order
    if (P.ok) {
        const int per_rb = U * R2;
        for (int rbl = warp; rbl < rb1 - rb0; rbl += kDecWarps) {
            const int w0 = owner(n2, kDecWarps, rbl * per_rb), w1 = owner(n2, kDecWarps, rbl * per_rb + per_rb - 1);
            if (w0 == w1) continue;   // whole in one warp: already stored
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int w = w0; w <= w1; w++) {
                int wa, wb;
                share(n2, w, kDecWarps, wa, wb);
                if (wa == wb) continue;
                const float4 v = part2[(w * 2 + (rbl == wa / per_rb ? 0 : 1)) * 32 + lane];
                s.x += v.x;
                s.y += v.y;
                s.z += v.z;
                s.w += v.w;
            }
            store_out(p, rb0 + rbl, s, g, q, bad2);
        }
    }
    warp_report(p, bad2, kNfOut);

    if (blockIdx.x == 0) publish_route(p, R);
}

template <int NPER>
__global__ void __launch_bounds__(kDecThreads, 1) decode_layer_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ DecRoute R;
    __shared__ DecPlan P;
    // Everything this layer reads may come from the previous kernel in the stream.
    grid_dep_wait();
    // this launch's barrier generation: no CTA can open the next one before every
    // CTA (this one included) has arrived, hence read it
    int gen = threadIdx.x == 0 ? *reinterpret_cast<volatile int32_t *>(p.dstate + kDsGen) : 0;
    __shared__ DecLayer W;
    if (threadIdx.x == 0)
        W = DecLayer{p.gate_codes, p.up_codes, p.gate_scales, p.up_scales, p.gate_global,
                     p.up_global, p.down_codes, p.down_scales, p.down_global, p.logits};
    __syncthreads();
    decode_body<NPER>(p, W, R, P, dsm, gen);
    // The next layer's grid may launch once every CTA is here.
    grid_dep_launch();
}

// A stack of decode layers in one launch over the FP32 residual stream
// (x <- x + layer_l(bf16(x)), in place): per layer its weights and router logits
// from the table, then a second grid barrier so that every row of x is final
// before the next layer reads it.
template <int NPER>
__global__ void __launch_bounds__(kDecThreads, 1) decode_stack_kernel(const Params p, const DecStack st) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ DecRoute R;
    __shared__ DecPlan P;
    grid_dep_wait();
    int gen = threadIdx.x == 0 ? *reinterpret_cast<volatile int32_t *>(p.dstate + kDsGen) : 0;
    __shared__ DecLayer W;
    // The parameters are read from shared memory inside the loop: values the
    // compiler would otherwise hoist out of it stay in registers across every
    // layer and spill.
    __shared__ Params Ps;
    if (threadIdx.x == 0) Ps = p;
#pragma unroll 1
    for (int l = 0; l < st.n; l++) {
        __syncthreads();   // every thread is done with the previous layer's W
        if (threadIdx.x == 0) {
            W = st.layer[l];
            W.logits = st.logits + (size_t)l * p.T * p.E;
        }
        __syncthreads();
        decode_body<NPER>(Ps, W, R, P, dsm, gen);
        if (!P.ok) break;   // a wait gave up (TIMEOUT latched): the rest is not run
        if (l + 1 < st.n && !grid_barrier(Ps, Ps.dstate, gen, 102, true, &P.ok)) break;
    }
    grid_dep_launch();
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

int decode_grid() { return sm_count(); }

// Dynamic shared memory: the gate/up phase's storage (F16 activation tile,
// split-granule parts) and the down phase's (every
// pair's h row, split-row-block parts) share one region; the routing scratch
// and every expert's three global scales follow. Kept well below the SM's 256 KB: L1 and shared memory share that
// storage, and the weight loads in flight need L1 room (a kernel holding over
// 200 KB of shared memory streamed about half as fast).
constexpr size_t kDecSmemMax = 150 * 1024;
constexpr size_t kPartBytes = (size_t)kDecWarps * 2 * 32 * 16;

static size_t decode_union_for(int T, int K, int H, int I) {
    const size_t ph1 = dec_xs_bytes(T, H) + kPartBytes;
    const size_t ph2 = (size_t)(T * K + 1) * dec_ld2(I) * 2 + kPartBytes;
    return ph1 > ph2 ? ph1 : ph2;
}
size_t decode_union_bytes(int T, int K, int H, int I) { return decode_union_for(T, K, H, I); }
static size_t decode_smem_for(int T, int K, int E, int H, int I) {
    return decode_union_for(T, K, H, I) + (size_t)5 * E * 4;
}

bool decode_fits(int H, int I, int K, int E) {
    if (H % 32 || I % 32) return false;
    return decode_smem_for(kSlots, K, E, H, I) <= kDecSmemMax;
}

template <int NPER>
static cudaError_t launch_layer(const Params &p, cudaStream_t s) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(decode_grid());
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = decode_smem_for(p.T, p.K, p.E, p.H, p.I);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_layer_kernel<NPER>, p);
}

template <int NPER>
static cudaError_t launch_stack(const Params &p, const DecStack &st, cudaStream_t s) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(decode_grid());
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = decode_smem_for(p.T, p.K, p.E, p.H, p.I);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_stack_kernel<NPER>, p, st);
}

// p: the stack's common parameters (the first layer's weights, which the
// kernel replaces per layer); layers / logits: the table.
cudaError_t launch_decode_stack(const Params &p, const DecLayerPtrs *layers, int n, const float *logits,
                                cudaStream_t s) {
    if (n < 1 || n > kMaxStackLayers) return cudaErrorInvalidValue;
    DecStack st{};
    st.n = n;
    st.logits = logits;
    for (int l = 0; l < n; l++) {
        const DecLayerPtrs &w = layers[l];
        st.layer[l] = DecLayer{w.gate_codes, w.up_codes, w.gate_scales, w.up_scales, w.gate_global,
                               w.up_global, w.down_codes, w.down_scales, w.down_global, nullptr};
    }
    const int nper = cdiv(p.E, 32);
    if (nper <= 1) return launch_stack<1>(p, st, s);
    if (nper <= 2) return launch_stack<2>(p, st, s);
    if (nper <= 4) return launch_stack<4>(p, st, s);
    if (nper <= 8) return launch_stack<8>(p, st, s);
    if (nper <= 16) return launch_stack<16>(p, st, s);
    return launch_stack<32>(p, st, s);
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
    // dynamic shared memory above the 48 KB default (the activations grow with H)
    const int big = (int)kDecSmemMax;
    const cudaError_t r[] = {
        cudaFuncSetAttribute(decode_stack_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_stack_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_stack_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_stack_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_stack_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
        cudaFuncSetAttribute(decode_stack_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, big),
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
