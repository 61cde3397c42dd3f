// Prefill grouped GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// One persistent CTA per SM walks a device-built tile list (expert, 128 output
// rows, up to 256 token pairs); no host read-back of counts ("Strata NVFP4"
// README, "How it differs from upstream Strata": one launch per expert group
// after one wait). Bigger prompt chunks re-stream each expert fewer times
// ("strata-5090-4070" README, "RAM: the one thing to know"), which is why a tile
// covers up to 256 pairs of one expert.
//
// Operands, per 64-wide K stage:
//   A (weights, M = 128 rows): dequantised by four warps from the packed planes
//     straight into the 128-byte-swizzled K-major layout. code x E4M3 scale is
//     exact in F16, so the MMA sees the stored weights without rounding. The
//     FP32 tensor scale is applied in the epilogue ("Strata NVFP4" README, "How
//     it differs": per-expert FP32 scales applied to each projection's output).
//   B (activations, N = pairs): the F16 copy of x (gate/up) or h (down) rows of
//     this expert's pairs, brought in by TMA with the same swizzle.
//   D (FP32, 128 lanes x N columns) in TMEM, double-buffered so the epilogue of
//     one tile overlaps the MMAs of the next.
// Epilogues: gate/up -> scales, SwiGLU, F16 h at the pair's position (64 gate
// rows and 64 up rows of the same intermediate indices share a tile, arranged
// so that each TMEM lane quarter holds 16 gate and the matching 16 up rows);
// down -> scale x routing weight, F16 row per pair (combined per token by a
// separate deterministic kernel).
//
// Warp roles (320 threads): 0-3 epilogue, 4-7 dequantise A, 8 TMA for B,
// 9 TMEM allocation + MMA issue. Every mbarrier wait is bounded (2 s); on
// give-up the CTA latches NVFP4_MOE_ERR_TIMEOUT, drains its own TMA and MMA
// work (bounded) and frees its TMEM before returning.
#include "common.cuh"

namespace nvmoe {

constexpr int kThreads = 320;
constexpr int kBM = 128;
constexpr int kAStage = kBM * kBK * 2;         // 16 KB
constexpr int kBStage = kBN * kBK * 2;         // 32 KB
constexpr int kBBox = 64;                      // rows per TMA box
constexpr int kTmemCols = 512;                 // two 256-column accumulators
constexpr int kStageBytes = 32 * kBM * 4;      // one epilogue staging buffer: 32 columns x 128 rows x FP32
// Both GEMMs: a 4-stage ring and one epilogue staging buffer (a 32-column chunk
// of h, or of the down projection's per-pair F16 rows).
template <int MODE> struct Cfg {
    static constexpr int stages = 4;
    static constexpr int bufs = 1;
};
constexpr int kPF = 4;                         // dequant loads in flight (k-steps)
constexpr uint64_t kDrainNs = 200000000ull;    // bounded drain on abort

struct __align__(8) Bars {
    uint64_t a_full[kStages];
    uint64_t b_full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_slot;
    int abort;
};

template <int MODE>
constexpr size_t smem_bytes() {
    return 1024 + Cfg<MODE>::stages * (kAStage + kBStage) + Cfg<MODE>::bufs * kStageBytes + sizeof(Bars);
}

// Iterates (tile, k-step) pairs of this CTA in order.
struct Cursor {
    int tl, kk, nk, ntl;
    __device__ Cursor(int nk_, int ntiles) : tl(0), kk(0), nk(nk_) {
        ntl = ntiles > (int)blockIdx.x ? cdiv(ntiles - (int)blockIdx.x, (int)gridDim.x) : 0;
    }
    __device__ bool valid() const { return tl < ntl; }
    __device__ int tile() const { return (int)blockIdx.x + tl * (int)gridDim.x; }
    __device__ void next() {
        if (++kk == nk) { kk = 0; ++tl; }
    }
};

template <int S>
struct Ring {
    int stage = 0;
    uint32_t phase = 0;
    __device__ void next() {
        if (++stage == S) { stage = 0; phase ^= 1; }
    }
};

template <int MODE>
__device__ inline void row_source(const Params &p, const Tile &t, int r, const uint8_t *&codes,
                                  const uint8_t *&scales) {
    if (MODE == 0) {
        const int q = r >> 5, l = r & 31;
        const int i = t.m0 + 16 * q + (l & 15);
        const size_t row = (size_t)t.expert * p.I + i;
        codes = (l < 16 ? p.gate_codes : p.up_codes) + row * (p.H / 2);
        scales = (l < 16 ? p.gate_scales : p.up_scales) + row * (p.H / 16);
    } else {
        const size_t row = (size_t)t.expert * p.H + t.m0 + r;
        codes = p.down_codes + row * (p.I / 2);
        scales = p.down_scales + row * (p.I / 16);
    }
}

struct StepData {
    uint4 c0, c1;
    uint32_t s;
};

__device__ inline StepData load_step(const uint8_t *codes, const uint8_t *scales, int kk) {
    StepData d;
    const uint4 *cp = reinterpret_cast<const uint4 *>(codes + 32 * kk);
    d.c0 = __ldg(cp);
    d.c1 = __ldg(cp + 1);
    d.s = __ldg(reinterpret_cast<const uint32_t *>(scales + 4 * kk));
    return d;
}

// Writes one 128-byte A row (64 F16 weights) in the 128B-swizzled layout.
__device__ inline void store_row(uint8_t *a_stage, int r, const StepData &d) {
    const uint32_t w[8] = {d.c0.x, d.c0.y, d.c0.z, d.c0.w, d.c1.x, d.c1.y, d.c1.z, d.c1.w};
    uint8_t *row = a_stage + r * 128;
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const uint32_t sc = e4m3_to_f16x2_bcast(d.s >> (8 * (j >> 1)));
        uint32_t o0, o1, o2, o3;
        e2m1x8_to_f16(w[j], o0, o1, o2, o3);
        uint4 v = make_uint4(hmul2(o0, sc), hmul2(o1, sc), hmul2(o2, sc), hmul2(o3, sc));
        *reinterpret_cast<uint4 *>(row + ((j ^ (r & 7)) << 4)) = v;
    }
}

// Named barrier over the four epilogue warps (ids 0 is __syncthreads).
__device__ inline void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const Params p, const __grid_constant__ CUtensorMap map_b) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *a_base = smem;
    constexpr int S = Cfg<MODE>::stages, NB = Cfg<MODE>::bufs;
    uint8_t *b_base = smem + S * kAStage;
    uint8_t *epi_stage = b_base + S * kBStage;                       // NB x kStageBytes
    Bars *bars = reinterpret_cast<Bars *>(epi_stage + NB * kStageBytes);
    volatile int *abort = &bars->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Tile *tiles = MODE == 0 ? p.tiles_gu : p.tiles_dn;
    const int ntiles = p.cnt[MODE == 0 ? kCntTilesGu : kCntTilesDn];
    const int Kdim = MODE == 0 ? p.H : p.I;
    const int nk = Kdim / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&bars->a_full[s], 128);
            mbar_init(&bars->b_full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 128);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(&bars->tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) tma_prefetch_desc(&map_b);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_slot;

    if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ dequantise A rows
        const int r = threadIdx.x - 128;
        Cursor ld(nk, ntiles), cs(nk, ntiles);
        Ring<S> ring;
        StepData q[kPF];
        int ld_tile = -1;
        const uint8_t *lcodes = nullptr, *lscales = nullptr;
#pragma unroll
        for (int j = 0; j < kPF; j++) {
            if (ld.valid()) {
                if (ld.tile() != ld_tile) {
                    ld_tile = ld.tile();
                    row_source<MODE>(p, tiles[ld_tile], r, lcodes, lscales);
                }
                q[j] = load_step(lcodes, lscales, ld.kk);
                ld.next();
            }
        }
        bool ok = true;
        while (ok && cs.valid()) {
#pragma unroll
            for (int j = 0; j < kPF; j++) {
                if (!ok || !cs.valid()) break;
                if (!mbar_wait(&bars->empty[ring.stage], ring.phase ^ 1, abort, p.status, 1)) {
                    ok = false;
                    break;
                }
                store_row(a_base + ring.stage * kAStage, r, q[j]);
                fence_proxy_async_smem();
                mbar_arrive(&bars->a_full[ring.stage]);
                ring.next();
                cs.next();
                if (ld.valid()) {
                    if (ld.tile() != ld_tile) {
                        ld_tile = ld.tile();
                        row_source<MODE>(p, tiles[ld_tile], r, lcodes, lscales);
                    }
                    q[j] = load_step(lcodes, lscales, ld.kk);
                    ld.next();
                }
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------ TMA for B
        // 64-row boxes of the pair-ordered B rows (F16 activations or h) into the
        // ring; the next tile's descriptor is read one tile ahead.
        if (lane == 0) {
            Cursor cs(nk, ntiles);
            Ring<S> ring;
            uint32_t issued = 0, issued_phase = 0;  // stages with a load in flight, their parity
            int cur_tile = -1;
            Tile t{}, t_n{};
            if (cs.valid()) t_n = tiles[cs.tile()];
            while (cs.valid()) {
                if (cs.tile() != cur_tile) {
                    cur_tile = cs.tile();
                    t = t_n;
                    if (cur_tile + (int)gridDim.x < ntiles) t_n = tiles[cur_tile + (int)gridDim.x];
                }
                if (!mbar_wait(&bars->empty[ring.stage], ring.phase ^ 1, abort, p.status, 2)) break;
                const int nbox = cdiv((t.ntok + 15) & ~15, kBBox);
                uint8_t *bs = b_base + ring.stage * kBStage;
                mbar_arrive_expect_tx(&bars->b_full[ring.stage], nbox * kBBox * kBK * 2);
                for (int b = 0; b < nbox; b++)
                    tma_load_2d(bs + b * kBBox * kBK * 2, &map_b, &bars->b_full[ring.stage],
                                cs.kk * kBK, t.pos0 + b * kBBox);
                issued |= 1u << ring.stage;
                issued_phase = (issued_phase & ~(1u << ring.stage)) | (ring.phase << ring.stage);
                ring.next();
                cs.next();
            }
            // Every stage's last load must have landed before this CTA may exit.
            for (int s = 0; s < S; s++)
                if (issued & (1u << s))
                    mbar_wait_drain(&bars->b_full[s], (issued_phase >> s) & 1, kDrainNs);
        }
    } else if (warp == 9) {
        // ----------------------------------------------------- MMA issue
        if (lane == 0) {
            Ring<S> ring;
            uint32_t acc_phase[2] = {0, 0};
            const int ntl = ntiles > (int)blockIdx.x ? cdiv(ntiles - (int)blockIdx.x, (int)gridDim.x) : 0;
            bool ok = true;
            for (int tl = 0; ok && tl < ntl; tl++) {
                const Tile t = tiles[(int)blockIdx.x + tl * (int)gridDim.x];
                const int buf = tl & 1;
                const int nmma = (t.ntok + 15) & ~15;
                const uint32_t idesc = idesc_f16(kBM, nmma);
                if (!mbar_wait(&bars->acc_empty[buf], acc_phase[buf] ^ 1, abort, p.status, 4)) break;
                acc_phase[buf] ^= 1;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * kBN;
                for (int kk = 0; kk < nk; kk++) {
                    if (!mbar_wait(&bars->a_full[ring.stage], ring.phase, abort, p.status, 5) ||
                        !mbar_wait(&bars->b_full[ring.stage], ring.phase, abort, p.status, 6)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t as = smem_u32(a_base + ring.stage * kAStage);
                    const uint32_t bs = smem_u32(b_base + ring.stage * kBStage);
#pragma unroll
                    for (int k16 = 0; k16 < kBK / 16; k16++)
                        tc_mma_f16(d_tmem, smem_desc_sw128(as + 32 * k16),
                                   smem_desc_sw128(bs + 32 * k16), idesc, (kk | k16) != 0);
                    tc_commit(&bars->empty[ring.stage]);
                    ring.next();
                }
                if (ok) tc_commit(&bars->acc_full[buf]);
            }
            // Drain: every MMA this thread issued completes before TMEM is freed.
            tc_commit(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, kDrainNs);
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int ntl = ntiles > (int)blockIdx.x ? cdiv(ntiles - (int)blockIdx.x, (int)gridDim.x) : 0;
        uint32_t acc_phase[2] = {0, 0};
        for (int tl = 0; tl < ntl; tl++) {
            const Tile t = tiles[(int)blockIdx.x + tl * (int)gridDim.x];
            const int buf = tl & 1;
            if (!mbar_wait(&bars->acc_full[buf], acc_phase[buf], abort, p.status, 8)) break;
            acc_phase[buf] ^= 1;
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * kBN + ((uint32_t)(warp * 32) << 16);
            const int e = t.expert;
            if (MODE == 0) {
                // SwiGLU; h staged as [32 columns][64 intermediates] F16, then written
                // with coalesced 16-byte stores (each column is 128 contiguous bytes of h).
                const float sg = p.gate_global[e], su = p.up_global[e];
                const int il = 16 * warp + (lane & 15);
                const bool is_gate = lane < 16;
                __half *hs = reinterpret_cast<__half *>(epi_stage);
                for (int c0 = 0; c0 < t.ntok; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tbase + c0, v);
                    const float xs_l = (c0 + lane < t.ntok) ? p.ps[t.pos0 + c0 + lane] : 0.0f;
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float mine_lo = __uint_as_float(v[j]);
                        const float mine_hi = __uint_as_float(v[16 + j]);
                        const float send = is_gate ? mine_hi : mine_lo;
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                        const float gacc = is_gate ? mine_lo : recv;
                        const float uacc = is_gate ? recv : mine_hi;
                        const int cj = j + (is_gate ? 0 : 16);
                        const float xs = __shfl_sync(0xffffffffu, xs_l, cj);
                        const float gv = gacc * sg * xs, uv = uacc * su * xs;
                        hs[cj * kGuRows + il] = __float2half_rn(silu(gv) * uv);
                    }
                    epi_sync();
                    const int ncol = min(32, t.ntok - c0);
                    for (int q = threadIdx.x; q < ncol * 8; q += 128) {
                        const int col = q >> 3, part = q & 7;
                        const uint4 val = reinterpret_cast<const uint4 *>(hs + col * kGuRows)[part];
                        reinterpret_cast<uint4 *>(p.h + (size_t)(t.pos0 + c0 + col) * p.I + t.m0)[part] = val;
                    }
                    epi_sync();
                }
            } else {
                // y * s_d * w staged as [32 columns][128 hidden rows] F16, written with
                // coalesced 16-byte stores into the pair's row of yp; the combine
                // kernel sums each token's K rows in a fixed order.
                const float sd = p.down_global[e];
                const int r = 32 * warp + lane;
                __half *ys = reinterpret_cast<__half *>(epi_stage);
                for (int c0 = 0; c0 < t.ntok; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tbase + c0, v);
                    const float w_l = (c0 + lane < t.ntok) ? p.pw[t.pos0 + c0 + lane] * sd : 0.0f;
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; j++)
                        ys[j * kBM + r] = __float2half_rn(__uint_as_float(v[j]) * __shfl_sync(0xffffffffu, w_l, j));
                    epi_sync();
                    const int ncol = min(32, t.ntok - c0);
                    for (int q = threadIdx.x; q < ncol * (kBM / 8); q += 128) {
                        const int col = q / (kBM / 8), part = q % (kBM / 8);
                        const uint4 val = reinterpret_cast<const uint4 *>(ys + col * kBM)[part];
                        reinterpret_cast<uint4 *>(p.xh + (size_t)(t.pos0 + c0 + col) * p.H + t.m0)[part] = val;
                    }
                    epi_sync();
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

cudaError_t prefill_init() {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<0>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes<0>());
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem_bytes<1>());
}

void launch_prefill_gemm(int mode, const Params &p, const CUtensorMap &map, int num_sms,
                         cudaStream_t s) {
    if (mode == 0)
        grouped_gemm_kernel<0><<<max(1, min(num_sms, p.max_tiles_gu)), kThreads, smem_bytes<0>(), s>>>(p, map);
    else
        grouped_gemm_kernel<1><<<max(1, min(num_sms, p.max_tiles_dn)), kThreads, smem_bytes<1>(), s>>>(p, map);
}

}  // namespace nvmoe
