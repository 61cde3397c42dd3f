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
// Larger batches: a tcgen05 GEMM, one CTA per (128 experts, 64 tokens) tile, two
// CTAs per SM (each hides the other's load latency).
// The tensor cores take BF16 operands, so each FP32 input is split exactly into
// three BF16 terms, x = x0 + x1 + x2 (x0 the nearest BF16 to x, x1 the nearest to
// x - x0, x2 = x - x0 - x1, which fits in BF16), and the tile runs three MMAs per
// K step into one FP32 accumulator: every product W * x_j is exact, the sums
// round in FP32, as in the small-batch kernel. BF16 activations need only x0.
// All 256 threads stage the operands (W_r rows copied, x split) into two
// 128-byte-swizzled K-major stages of 64 K; one thread issues the MMAs and
// commits each stage to an mbarrier that frees it; warps 0..3 read the 128 x 64
// accumulator out of TMEM.
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
    const int xbytes = T * p.H * act_elem_bytes(p.act_type);
    for (int c = threadIdx.x; c < xbytes / 16; c += blockDim.x)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(rv_xs + 16 * c)),
                     "l"(static_cast<const uint8_t *>(p.act) + 16 * c)
                     : "memory");
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
constexpr int kRtM = 128;        // experts per CTA (TMEM lanes)
constexpr int kRtN = 64;         // tokens per CTA (accumulator columns)
constexpr int kRtK = 64;         // K per stage: 128 bytes of BF16 per row
constexpr int kRtThreads = 256;
constexpr int kRtTileA = kRtM * kRtK * 2;        // 16 KB: 128 W_r rows x 128 B
constexpr int kRtTileB = kRtN * kRtK * 2;        // 8 KB: 64 token rows x 128 B
constexpr int kRtStage = kRtTileA + 3 * kRtTileB; // A, then the three parts of x
constexpr int kRtSmem = 2 * kRtStage + 1024 + 64; // two stages, 1024-B alignment slack, barriers
constexpr int kRtChunksA = kRtM * 8 / kRtThreads; // 16-byte A chunks per thread per stage (4)
constexpr int kRtChunksB = kRtN * 8 / kRtThreads; // 8-input x chunks per thread per stage (2)
constexpr uint64_t kRtWaitNs = 2000000000ull;

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

// One thread's share of a K stage: 16-byte A chunks (8 BF16 of a W_r row) and
// x chunks (8 inputs of a token), loaded into registers one stage ahead.
struct RtRegs {
    uint4 a[kRtChunksA];
    float x[kRtChunksB][8];
};

__device__ inline void rt_load(const Params &p, int m0, int n0, int k0, RtRegs &r) {
#pragma unroll
    for (int i = 0; i < kRtChunksA; i++) {
        const int c = threadIdx.x + kRtThreads * i;   // row c / 8, chunk c % 8
        const int row = c >> 3, k = k0 + 8 * (c & 7), e = m0 + row;
        r.a[i] = (e < p.E && k < p.H)
                     ? __ldg(reinterpret_cast<const uint4 *>(p.router_w + (size_t)e * p.H + k))
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kRtChunksB; i++) {
        const int c = threadIdx.x + kRtThreads * i;
        const int row = c >> 3, k = k0 + 8 * (c & 7), t = n0 + row;
        if (t < p.T && k < p.H) {
            router_x8(p, t, k / 8, r.x[i]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; j++) r.x[i][j] = 0.0f;
        }
    }
}

// Stores the registers into stage `st` in the 128-byte swizzled K-major layout
// (16-byte chunk c of row r at r * 128 + ((c ^ (r & 7)) << 4)).
__device__ inline void rt_store(uint8_t *st, const RtRegs &r, int nsplit) {
#pragma unroll
    for (int i = 0; i < kRtChunksA; i++) {
        const int c = threadIdx.x + kRtThreads * i;
        const int row = c >> 3, ch = c & 7;
        *reinterpret_cast<uint4 *>(st + row * 128 + ((ch ^ (row & 7)) << 4)) = r.a[i];
    }
#pragma unroll
    for (int i = 0; i < kRtChunksB; i++) {
        const int c = threadIdx.x + kRtThreads * i;
        const int row = c >> 3, ch = c & 7;
        const int off = kRtTileA + row * 128 + ((ch ^ (row & 7)) << 4);
        uint32_t w[3][4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            uint32_t l0, l1, l2, h0, h1, h2;
            split3(r.x[i][2 * j], l0, l1, l2);
            split3(r.x[i][2 * j + 1], h0, h1, h2);
            w[0][j] = l0 | (h0 << 16);
            w[1][j] = l1 | (h1 << 16);
            w[2][j] = l2 | (h2 << 16);
        }
#pragma unroll
        for (int sp = 0; sp < 3; sp++)
            if (sp < nsplit)
                *reinterpret_cast<uint4 *>(st + off + sp * kRtTileB) =
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

__global__ void __launch_bounds__(kRtThreads, 2) router_gemm_kernel(Params p) {
    extern __shared__ uint8_t rt_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rt_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 2 * kRtStage);   // [0..1] stage free, [2] drain
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4);
    __shared__ int s_ok;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kRtM, n0 = blockIdx.y * kRtN;
    const int nsplit = p.act_type == NVFP4_MOE_ACT_BF16 ? 1 : 3;
    const int nk = cdiv(p.H, kRtK);

    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        fence_barrier_init();
        s_ok = 1;
    }
    if (warp == 0) {
        tmem_alloc1(tmem_slot, kRtN);
        tmem_relinquish1();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t idesc = idesc_bf16(kRtM, kRtN);

    // two register sets in turn: the loads of stage ks + 1 are in flight while
    // stage ks is stored and multiplied
    RtRegs r0, r1;
    rt_load(p, m0, n0, 0, r0);
    int ks = 0;
    auto step = [&](RtRegs &cur, RtRegs &nxt) {
        const int s = ks & 1;
        uint8_t *st = sm + s * kRtStage;
        if (ks + 1 < nk) rt_load(p, m0, n0, (ks + 1) * kRtK, nxt);
        if (ks >= 2 && threadIdx.x == 0 && s_ok)   // the MMAs of step ks - 2 are done with stage s
            s_ok = rt_wait(&bars[s], ((ks >> 1) - 1) & 1, p.status, 201);
        __syncthreads();
        if (!s_ok) return;
        rt_store(st, cur, nsplit);
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint32_t as = smem_u32(st);
#pragma unroll
            for (int k16 = 0; k16 < kRtK / 16; k16++)
                for (int sp = 0; sp < nsplit; sp++)
                    tc_mma_bf16(tmem, smem_desc_sw128(as + 32 * k16),
                                smem_desc_sw128(as + kRtTileA + sp * kRtTileB + 32 * k16), idesc,
                                (ks | k16 | sp) != 0);
            tc_commit1(&bars[s]);
        }
        ks++;
    };
    while (ks < nk && s_ok) {
        step(r0, r1);
        if (ks >= nk || !s_ok) break;
        step(r1, r0);
    }
    // every MMA issued so far has completed once the drain barrier fires
    if (threadIdx.x == 0) {
        tc_commit1(&bars[2]);
        if (!rt_wait(&bars[2], 0, p.status, 202)) s_ok = 0;
    }
    __syncthreads();
    tc_fence_after();
    if (warp < 4 && s_ok) {
        const int e = m0 + 32 * warp + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < kRtN; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + c0, v);
            tmem_ld_wait();
            if (e < p.E) {
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const int t = n0 + c0 + j;
                    if (t < p.T) p.rlogits[(size_t)t * p.E + e] = __uint_as_float(v[j]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc1(tmem, kRtN);
}

cudaError_t launch_router(const Params &p, cudaStream_t s) {
    const size_t xbytes = (size_t)p.T * p.H * act_elem_bytes(p.act_type);
    if (p.T <= kRvMaxT && xbytes <= kRvSmemMax) {
        router_gemv_kernel<<<cdiv(p.E, kRvWarps), kRvWarps * 32, xbytes, s>>>(p);
        return cudaGetLastError();
    }
    const dim3 grid(cdiv(p.E, kRtM), cdiv(p.T, kRtN));
    router_gemm_kernel<<<grid, kRtThreads, kRtSmem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t router_init() {
    const cudaError_t a =
        cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRtSmem);
    const cudaError_t b =
        cudaFuncSetAttribute(router_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRvSmemMax);
    return a != cudaSuccess ? a : b;
}

}  // namespace nvmoe
