// Router projection: logits[T][E] = x[T][H] . W_r[E][H]^T, ahead of the routing.
//
// The pages keep the router's BF16 projection on FP32-exact inputs ("Strata
// NVFP4" README, "How it differs from upstream Strata": the prompt path's BF16
// projections -- router, indexer, gates -- take FP32-exact inputs). So x, the
// layer's input as FP32 (BF16 and FP32 activations as given, int8 ones as the
// FP32 product q * scale), is never rounded to BF16 here.
//
// Small batches (T <= 8): one warp per expert, FP32 fused multiply-adds (the
// product of a BF16 weight and an FP32 input is exact inside the FMA; only the
// sum rounds), lanes reduced in a fixed tree.
//
// Larger batches: a tcgen05 GEMM, one CTA per 64 tokens against up to 512
// experts (four 128-row accumulators in TMEM; 256 for FP32 / int8 inputs), so a
// token's activations are read once or twice.
// The tensor cores take BF16 operands, so each FP32 input is split exactly into
// three BF16 terms, x = x0 + x1 + x2 (x0 the nearest BF16 to x, x1 the nearest to
// x - x0, x2 = x - x0 - x1, which fits in BF16), and the tile runs three MMAs per
// K step into one FP32 accumulator: every product W * x_j is exact, the sums
// round in FP32, as in the small-batch kernel. BF16 activations need only x0.
// The operands reach shared memory by cp.async, in a ring of two or three
// 128-byte-swizzled K-major stages of 64 K (BF16 activations straight into their
// tile; FP32 / int8 ones raw, then split by all 256 threads); one thread issues
// the MMAs and commits each stage to an mbarrier that frees it; warps 0..3 read
// the accumulators out of TMEM.
#include "common.cuh"

namespace nvmoe {

// Eight consecutive router inputs k8*8.. of token t as FP32 (BF16 / FP32 as
// given, int8 as q * scale).
__device__ inline void router_x8(const Params &p, int t, int k8, float (&v)[8]) {
    const size_t off = (size_t)t * p.H + 8 * k8;
    if (p.act_type == NVFP4_MOE_ACT_BF16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.act) + off));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else if (p.act_type == NVFP4_MOE_ACT_INT8) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(static_cast<const int8_t *>(p.act) + off));
        const uint32_t w[2] = {u.x, u.y};
        const float s = __ldg(p.act_scale + t);
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = __fmul_rn((float)(int8_t)(w[i >> 2] >> (8 * (i & 3))), s);
    } else {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p.act) + off));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p.act) + off) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

__device__ inline float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ inline float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------ small batches
constexpr int kRvWarps = 4;
constexpr int kRvMaxT = NVFP4_MOE_DECODE_MAX_T;
constexpr int kRvChunks = 8;     // 16-byte weight chunks a lane loads per batch (256 weights)
constexpr size_t kRvSmemMax = 96 * 1024;   // staged activation rows; larger batches take the GEMM

// Activation bytes per element as the layer receives them.
__host__ __device__ inline int act_elem_bytes(int act_type) {
    return act_type == NVFP4_MOE_ACT_BF16 ? 2 : (act_type == NVFP4_MOE_ACT_INT8 ? 1 : 4);
}

// Eight router inputs of token t from the raw activation rows staged in shared
// memory (same conversions as router_x8).
__device__ inline void router_x8_smem(const Params &p, const uint8_t *xs, int t, int k8, float (&v)[8]) {
    if (p.act_type == NVFP4_MOE_ACT_BF16) {
        const uint4 u = reinterpret_cast<const uint4 *>(xs + (size_t)t * p.H * 2)[k8];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else if (p.act_type == NVFP4_MOE_ACT_INT8) {
        const uint2 u = reinterpret_cast<const uint2 *>(xs + (size_t)t * p.H)[k8];
        const uint32_t w[2] = {u.x, u.y};
        const float s = __ldg(p.act_scale + t);
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = __fmul_rn((float)(int8_t)(w[i >> 2] >> (8 * (i & 3))), s);
    } else {
        const float4 a = reinterpret_cast<const float4 *>(xs + (size_t)t * p.H * 4)[2 * k8];
        const float4 b = reinterpret_cast<const float4 *>(xs + (size_t)t * p.H * 4)[2 * k8 + 1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// One warp per expert. The T activation rows go to shared memory by cp.async
// while each warp's weight chunks are already loading; then FP32 fused
// multiply-adds (exact products, rounded sums) and a fixed lane tree.
__global__ void __launch_bounds__(kRvWarps * 32) router_gemv_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t rv_xs[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kRvWarps + warp;
    const int T = p.T, n8 = p.H / 8;
    const int xbytes = T * p.H * act_elem_bytes(p.act_type), nx = xbytes / 16;
    // every CTA copies the same rows: each starts at its own piece and wraps
    const int x_first = (int)(((long long)blockIdx.x * 97) % nx);
    for (int i = threadIdx.x; i < nx; i += blockDim.x) {
        const int c = (i + x_first) % nx;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(rv_xs + 16 * c)),
                     "l"(static_cast<const uint8_t *>(p.act) + 16 * c)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    float acc[kRvMaxT];
#pragma unroll
    for (int t = 0; t < kRvMaxT; t++) acc[t] = 0.0f;
    const uint4 *wr = reinterpret_cast<const uint4 *>(p.router_w + (size_t)(e < p.E ? e : 0) * p.H);
    bool first = true;
    for (int base = 0; base < n8; base += 32 * kRvChunks) {
        uint4 wv[kRvChunks];
#pragma unroll
        for (int i = 0; i < kRvChunks; i++) {
            const int k8 = base + lane + 32 * i;
            wv[i] = (e < p.E && k8 < n8) ? __ldg(wr + k8) : make_uint4(0, 0, 0, 0);
        }
        if (first) {
            asm volatile("cp.async.wait_all;" ::: "memory");
            __syncthreads();
            first = false;
        }
#pragma unroll
        for (int i = 0; i < kRvChunks; i++) {
            const int k8 = base + lane + 32 * i;
            if (k8 < n8) {
                const float w8[8] = {bf16_lo(wv[i].x), bf16_hi(wv[i].x), bf16_lo(wv[i].y), bf16_hi(wv[i].y),
                                     bf16_lo(wv[i].z), bf16_hi(wv[i].z), bf16_lo(wv[i].w), bf16_hi(wv[i].w)};
#pragma unroll
                for (int t = 0; t < kRvMaxT; t++) {
                    if (t < T) {
                        float x8[8];
                        router_x8_smem(p, rv_xs, t, k8, x8);
#pragma unroll
                        for (int j = 0; j < 8; j++) acc[t] = __fmaf_rn(w8[j], x8[j], acc[t]);
                    }
                }
            }
        }
    }
    if (first) {   // n8 == 0 cannot happen (H >= 32), but every thread must pass the barrier
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
    }
#pragma unroll
    for (int t = 0; t < kRvMaxT; t++) {
        if (t < T) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && e < p.E) p.rlogits[(size_t)t * p.E + e] = v;
        }
    }
}

// ------------------------------------------------------------------ GEMM
// 128-expert M tiles per CTA: four (512 experts) for BF16 activations, two for
// FP32 / int8 ones (whose stages also hold the raw rows and three part tiles),
// so that three stages fit; more experts -> more CTAs along grid.y.
__host__ __device__ inline int rt_mt_max(int act_type) { return act_type == NVFP4_MOE_ACT_BF16 ? 4 : 2; }
constexpr int kRtN = 64;         // tokens per CTA (accumulator columns per M tile)
constexpr int kRtK = 64;         // K per stage: 128 bytes of BF16 per row
constexpr int kRtThreads = 256;
constexpr int kRtTileA = 128 * kRtK * 2;         // 16 KB: 128 W_r rows x 128 B
constexpr int kRtTileB = kRtN * kRtK * 2;        // 8 KB: 64 token rows x 128 B
constexpr int kRtSmemBudget = 216 * 1024;        // stages of the ring (the rest: barriers, alignment)
constexpr uint64_t kRtWaitNs = 2000000000ull;

// Bytes of one stage: A tiles, the x part tiles, and (FP32 / int8 inputs) the raw
// activations the parts are split from.
__host__ __device__ inline int rt_raw_bytes(int act_type) {
    return act_type == NVFP4_MOE_ACT_BF16 ? 0 : kRtN * kRtK * (act_type == NVFP4_MOE_ACT_INT8 ? 1 : 4);
}
__host__ __device__ inline int rt_stage_bytes(int mt, int act_type) {
    const int nsplit = act_type == NVFP4_MOE_ACT_BF16 ? 1 : 3;
    return mt * kRtTileA + nsplit * kRtTileB + rt_raw_bytes(act_type);
}
__host__ __device__ inline int rt_stages(int mt, int act_type) {
    const int n = kRtSmemBudget / rt_stage_bytes(mt, act_type);
    return n < 3 ? n : 3;
}

__device__ inline void tmem_alloc1(uint32_t *slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot_smem)),
                 "r"(ncols));
}
__device__ inline void tmem_relinquish1() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ inline void tmem_dealloc1(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ inline void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                   uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ inline void tc_commit1(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// kind::f16 instruction descriptor with BF16 A and B, F32 accumulation, K-major.
__host__ __device__ inline uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// 16-byte asynchronous copy; src_bytes = 0 fills the destination with zeros.
__device__ inline void cp16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}

// x = x0 + x1 + x2 exactly, each a BF16 (bits returned).
__device__ inline void split3(float x, uint32_t &b0, uint32_t &b1, uint32_t &b2) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h0);          // exact: x and h0 share the leading bits
    const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(h1);         // exact, and at most 8 significant bits
    const __nv_bfloat16 h2 = __float2bfloat16_rn(r2);   // = r2
    b0 = __bfloat16_as_ushort(h0);
    b1 = __bfloat16_as_ushort(h1);
    b2 = __bfloat16_as_ushort(h2);
}

// Swizzled offset (128-byte rows, 16-byte chunk c of row r at c ^ (r & 7)).
__device__ inline int swz(int row, int ch) { return row * 128 + ((ch ^ (row & 7)) << 4); }

// Issues the copies of K step k0 into a stage: the CTA's W_r rows (zeros past E
// or H) and the tokens' activations -- straight into the BF16 part tile, or raw
// (FP32 / int8) for the split.
__device__ inline void rt_issue(const Params &p, uint8_t *st, int mt, int m0, int n0, int k0) {
    for (int c = threadIdx.x; c < mt * 128 * 8; c += kRtThreads) {
        const int row = c >> 3, ch = c & 7, e = m0 + row, k = k0 + 8 * ch;
        const bool ok = e < p.E && k < p.H;
        cp16(st + (row >> 7) * kRtTileA + swz(row & 127, ch),
             p.router_w + (ok ? (size_t)e * p.H + k : 0), ok ? 16 : 0);
    }
    uint8_t *bt = st + mt * kRtTileA;
    if (p.act_type == NVFP4_MOE_ACT_BF16) {
        for (int c = threadIdx.x; c < kRtN * 8; c += kRtThreads) {
            const int row = c >> 3, ch = c & 7, t = n0 + row, k = k0 + 8 * ch;
            const bool ok = t < p.T && k < p.H;
            cp16(bt + swz(row, ch), static_cast<const __nv_bfloat16 *>(p.act) + (ok ? (size_t)t * p.H + k : 0),
                 ok ? 16 : 0);
        }
    } else {
        // raw rows: kRtK elements of each token, 16-byte pieces
        const int eb = p.act_type == NVFP4_MOE_ACT_INT8 ? 1 : 4, per = kRtK * eb / 16;
        uint8_t *raw = bt + 3 * kRtTileB;
        for (int c = threadIdx.x; c < kRtN * per; c += kRtThreads) {
            const int row = c / per, piece = c - row * per, t = n0 + row;
            const int k = k0 + piece * 16 / eb;
            const bool ok = t < p.T && k < p.H;
            cp16(raw + row * kRtK * eb + 16 * piece,
                 static_cast<const uint8_t *>(p.act) + (ok ? ((size_t)t * p.H + k) * eb : 0), ok ? 16 : 0);
        }
    }
}

// FP32 / int8 stages: the raw activations -> the three exact BF16 part tiles.
__device__ inline void rt_split(const Params &p, uint8_t *st, int mt, int n0) {
    uint8_t *bt = st + mt * kRtTileA;
    const uint8_t *raw = bt + 3 * kRtTileB;
    for (int c = threadIdx.x; c < kRtN * 8; c += kRtThreads) {
        const int row = c >> 3, ch = c & 7;
        float v[8];
        if (p.act_type == NVFP4_MOE_ACT_INT8) {
            const uint2 u = reinterpret_cast<const uint2 *>(raw + row * kRtK)[ch];
            const uint32_t w[2] = {u.x, u.y};
            const int t = n0 + row;
            const float s = t < p.T ? __ldg(p.act_scale + t) : 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) v[i] = __fmul_rn((float)(int8_t)(w[i >> 2] >> (8 * (i & 3))), s);
        } else {
            const float4 a = reinterpret_cast<const float4 *>(raw + row * kRtK * 4)[2 * ch];
            const float4 b = reinterpret_cast<const float4 *>(raw + row * kRtK * 4)[2 * ch + 1];
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        uint32_t w[3][4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            uint32_t l0, l1, l2, h0, h1, h2;
            split3(v[2 * j], l0, l1, l2);
            split3(v[2 * j + 1], h0, h1, h2);
            w[0][j] = l0 | (h0 << 16);
            w[1][j] = l1 | (h1 << 16);
            w[2][j] = l2 | (h2 << 16);
        }
#pragma unroll
        for (int sp = 0; sp < 3; sp++)
            *reinterpret_cast<uint4 *>(bt + sp * kRtTileB + swz(row, ch)) =
                make_uint4(w[sp][0], w[sp][1], w[sp][2], w[sp][3]);
    }
}

// Bounded wait on an mbarrier phase; latches TIMEOUT and returns false on give-up.
__device__ inline bool rt_wait(uint64_t *bar, uint32_t parity, int32_t *status, int where) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kRtWaitNs) {
            latch_status(status, NVFP4_MOE_ERR_TIMEOUT, where);
            return false;
        }
    }
    return true;
}

// One CTA: tokens [n0, n0 + 64) against up to 4 x 128 experts from m0. A ring of
// `ns` stages is filled by cp.async (ns - 1 K steps ahead); the stage of step
// ks - 1 is refilled once its MMAs have completed.
__global__ void __launch_bounds__(kRtThreads, 1) router_gemm_kernel(Params p) {
    extern __shared__ uint8_t rt_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rt_smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mtx = rt_mt_max(p.act_type);
    const int n0 = blockIdx.x * kRtN, m0 = blockIdx.y * mtx * 128;
    const int mt = min(mtx, cdiv(p.E - m0, 128));
    const int nsplit = p.act_type == NVFP4_MOE_ACT_BF16 ? 1 : 3;
    const int sb = rt_stage_bytes(mt, p.act_type), ns = rt_stages(mt, p.act_type);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ns * sb);   // [0..ns) stage's MMAs done, [3] drain
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);
    __shared__ int s_ok;
    const int nk = cdiv(p.H, kRtK);
    const uint32_t ncols = mt * kRtN <= 64 ? 64 : (mt * kRtN <= 128 ? 128 : 256);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; i++) mbar_init(&bars[i], 1);
        fence_barrier_init();
        s_ok = 1;
    }
    if (warp == 0) {
        tmem_alloc1(tmem_slot, ncols);
        tmem_relinquish1();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = idesc_bf16(128, kRtN);

    // Every CTA reads the same W_r rows; each starts its sweep over K at its own
    // step (and wraps), so that the CTAs do not all ask for the same lines at once.
    const int k_first = (int)(((long long)blockIdx.x * 7 + blockIdx.y * 3) % nk);
    auto kstep = [&](int j) { return (k_first + j) % nk; };
    for (int j = 0; j < ns - 1; j++) {
        if (j < nk) rt_issue(p, sm + j * sb, mt, m0, n0, kstep(j) * kRtK);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int ks = 0; ks < nk; ks++) {
        const int s = ks % ns;
        uint8_t *st = sm + s * sb;
        // this step's copies (one group committed per step; ns - 2 may stay in flight)
        if (ns == 3) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        if (nsplit == 3) {
            rt_split(p, st, mt, n0);
            __syncthreads();
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint32_t as = smem_u32(st), bs = as + mt * kRtTileA;
            for (int j = 0; j < mt; j++)
#pragma unroll
                for (int k16 = 0; k16 < kRtK / 16; k16++)
                    for (int sp = 0; sp < nsplit; sp++)
                        tc_mma_bf16(tmem + j * kRtN, smem_desc_sw128(as + j * kRtTileA + 32 * k16),
                                    smem_desc_sw128(bs + sp * kRtTileB + 32 * k16), idesc,
                                    (ks | k16 | sp) != 0);
            tc_commit1(&bars[s]);
            // the stage of step ks - 1 is refilled (for step ks + ns - 1) once its MMAs are done
            if (ks >= 1 && s_ok) {
                const int ps = (ks - 1) % ns, use = (ks - 1) / ns;
                s_ok = rt_wait(&bars[ps], use & 1, p.status, 201);
            }
        }
        __syncthreads();
        if (!s_ok) break;
        const int kn = ks + ns - 1;
        if (kn < nk) rt_issue(p, sm + (kn % ns) * sb, mt, m0, n0, kstep(kn) * kRtK);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // every MMA issued so far has completed once the drain barrier fires
    if (threadIdx.x == 0) {
        tc_commit1(&bars[3]);
        if (!rt_wait(&bars[3], 0, p.status, 202)) s_ok = 0;
    }
    __syncthreads();
    tc_fence_after();
    if (warp < 4 && s_ok) {
        for (int j = 0; j < mt; j++) {
            const int e = m0 + 128 * j + 32 * warp + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < kRtN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + j * kRtN + c0, v);
                tmem_ld_wait();
                if (e < p.E) {
#pragma unroll
                    for (int q = 0; q < 32; q++) {
                        const int t = n0 + c0 + q;
                        if (t < p.T) p.rlogits[(size_t)t * p.E + e] = __uint_as_float(v[q]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc1(tmem, ncols);
}

static size_t rt_smem_for(int E, int act_type) {
    const int mtx = rt_mt_max(act_type);
    const int mt = E < mtx * 128 ? cdiv(E, 128) : mtx;
    return (size_t)rt_stages(mt, act_type) * rt_stage_bytes(mt, act_type) + 1024 + 64;
}

cudaError_t launch_router(const Params &p, cudaStream_t s) {
    const size_t xbytes = (size_t)p.T * p.H * act_elem_bytes(p.act_type);
    if (p.T <= kRvMaxT && xbytes <= kRvSmemMax) {
        router_gemv_kernel<<<cdiv(p.E, kRvWarps), kRvWarps * 32, xbytes, s>>>(p);
        return cudaGetLastError();
    }
    const dim3 grid(cdiv(p.T, kRtN), cdiv(p.E, rt_mt_max(p.act_type) * 128));
    router_gemm_kernel<<<grid, kRtThreads, rt_smem_for(p.E, p.act_type), s>>>(p);
    return cudaGetLastError();
}

cudaError_t router_init() {
    const cudaError_t a =
        cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kRtSmemBudget + 1024 + 64);
    const cudaError_t b =
        cudaFuncSetAttribute(router_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRvSmemMax);
    return a != cudaSuccess ? a : b;
}

}  // namespace nvmoe
