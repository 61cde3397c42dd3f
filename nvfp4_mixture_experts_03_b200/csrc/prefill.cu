// Prefill grouped GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// computed by pairs of CTAs (clusters of two, one M = 256 pair MMA per K step).
//
// One persistent CTA pair walks a device-built tile list (expert, 256 output
// rows, up to 256 token pairs); no host read-back of counts ("Strata NVFP4"
// README, "How it differs from upstream Strata": one launch per expert group
// after one wait). Bigger prompt chunks re-stream each expert fewer times
// ("strata-5090-4070" README, "RAM: the one thing to know"), which is why a tile
// covers up to 256 pairs of one expert.
//
// Operands, per ring stage of 128 K (two 64-wide K blocks), in each CTA of the
// pair:
//   A (weights, 128 of the tile's 256 rows): dequantised by eight warps from the
//     packed planes straight into the 128-byte-swizzled K-major layout. code x
//     E4M3 scale is exact in F16, so the MMA sees the stored weights without
//     rounding. The FP32 tensor scale is applied in the epilogue ("Strata NVFP4"
//     README, "How it differs": per-expert FP32 scales applied to each
//     projection's output).
//   B (activations): half of the tile's pair rows (the F16 copy of x for
//     gate/up, h for down), brought in by TMA with the same swizzle; the bytes
//     of both halves are counted on the leader CTA's barrier.
//   D (FP32, this CTA's 128 rows x N columns) in its own TMEM, double-buffered so
//     the epilogue of one tile overlaps the MMAs of the next.
// The leader CTA issues the pair MMAs; their completions are multicast to both
// CTAs. Compared with one CTA per 128-row tile, each SM streams half the B bytes
// per MMA and the tensor cores read each B row once for 256 weight rows.
// Epilogues: gate/up -> scales, SwiGLU, F16 h at the pair's position (each CTA
// owns 64 intermediates: 64 gate rows and the 64 matching up rows, arranged so
// that each TMEM lane quarter holds 16 gate and the matching 16 up rows);
// down -> scale x routing weight, F16 row per pair (whole 32-pair chunks leave
// by one bulk tensor store; combined per token by a separate deterministic
// kernel).
//
// Warp roles (480 threads per CTA): 0-3 epilogue, 4-11 dequantise A (two threads
// per row: one for each half of every 64-wide K block), 12 TMA for B, 13 TMEM
// allocation (+ MMA issue in the leader), 14 raw weight stages (codes by TMA,
// scales by cp.async, 4 K steps per stage) so the dequant warps read only
// shared memory. Every mbarrier wait is bounded
// (2 s); on give-up the CTA latches NVFP4_MOE_ERR_TIMEOUT, drains what it can,
// lets in-flight copies land, and both CTAs free their TMEM after a cluster
// barrier.
#include "common.cuh"

namespace nvmoe {

constexpr int kThreads = 480;
constexpr int kBM = 128;                       // A rows per CTA (the pair MMA has M = 256)
constexpr int kGuCta = kGuRows / 2;            // intermediates per CTA in a gate/up tile
constexpr int kBRows = kBN / 2;                // B rows per CTA
constexpr int kSub = 2;                        // 64-wide K blocks (one 128-byte swizzle row each) per stage
constexpr int kSubBytes = kBM * kBK * 2;       // 16 KB: one block of A (or of B) per CTA
constexpr int kAStage = kSub * kSubBytes;      // 32 KB: 128 K of A
constexpr int kBStage = kSub * kBRows * kBK * 2;   // 32 KB: 128 K of B
constexpr int kBBox = 64;                      // rows per TMA box
constexpr int kBoxBytes = kBBox * kBK * 2;     // 8 KB
constexpr int kRing = 2;                       // A/B pipeline stages of 128 K (eight MMAs each)
constexpr int kRawSteps = 4;                   // K steps per raw weight stage
constexpr int kRawStages = 4;                  // 16 K steps of weights in flight: covers HBM latency
constexpr int kRawCodeBytes = kBM * kRawSteps * 32;   // 128 rows x 128 B of E2M1 codes
constexpr int kRawScaleBytes = kBM * kRawSteps * 4;   // 128 rows x 16 B of E4M3 scales
constexpr int kRawBytes = kRawCodeBytes + kRawScaleBytes;
static_assert(kRawSteps % kSub == 0 && kBRows * kBK * 2 == kSubBytes, "a raw stage holds whole ring stages");
constexpr int kTmemCols = 512;                 // two 256-column accumulators
constexpr int kEpiBytes = 2 * 32 * kBM * 2;    // epilogue staging: 2 x (32 columns x 128 rows x F16)
constexpr int kColBytes = kBN * 4;            // one per-column factor array of a tile (FP32)
constexpr uint64_t kDrainNs = 200000000ull;    // bounded drain on abort
constexpr uint64_t kSettleNs = 1000000ull;     // lets in-flight copies land after an abort
constexpr uint16_t kBothCtas = 0x3;

struct __align__(8) Bars {
    uint64_t a_full[kRing];     // leader: 8 dequant warps x 2 CTAs, and the B warp's expect_tx
                                //   for both halves of B (one barrier per stage for the MMA)
    uint64_t empty[kRing];      // both: the pair MMA's commit
    uint64_t raw_full[kRawStages];   // code bytes (TMA) + 32 scale-copy lanes
    uint64_t raw_empty[kRawStages];  // 8 dequant warps
    uint64_t acc_full[2];       // both: the pair MMA's commit
    uint64_t acc_empty[2];      // leader: 4 epilogue warps x 2 CTAs
    uint64_t drain;
    uint32_t tmem_slot;
    int abort;
};

constexpr size_t smem_bytes() {
    return 1024 + kRing * (kAStage + kBStage) + kRawStages * kRawBytes + kEpiBytes + 2 * kColBytes +
           sizeof(Bars);
}

// Iterates (tile, k-step) pairs of this CTA pair in order.
struct Cursor {
    int tl, kk, nk, ntl, cid, ncl;
    __device__ Cursor(int nk_, int ntiles, int cid_, int ncl_)
        : tl(0), kk(0), nk(nk_), cid(cid_), ncl(ncl_) {
        ntl = ntiles > cid ? cdiv(ntiles - cid, ncl) : 0;
    }
    __device__ bool valid() const { return tl < ntl; }
    __device__ int tile() const { return cid + tl * ncl; }
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

// First weight row of this CTA's 128-row half of tile t (down: the second half of
// the last tile lies past H when H % 256 == 128; it then reads the first half's
// rows, in bounds, and its results are dropped).
// Bulk tensor store of a shared-memory box (no swizzle) to global, in this
// thread's bulk group; commit and waits for the groups this thread issued.
__device__ inline void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ inline void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// all but the newest group have finished reading their shared memory
__device__ inline void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every group has completed (its global writes done)
__device__ inline void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Non-blocking test: has the phase with this parity completed?
__device__ inline bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

template <int MODE>
__device__ inline int half_row0(const Params &p, const Tile &t, int rank) {
    if (MODE == 0) return t.expert * p.I + t.m0 + kGuCta * rank;
    const int m = t.m0 + kBM * rank < p.H ? t.m0 + kBM * rank : t.m0;
    return t.expert * p.H + m;
}

// Where A row r (0..127) of the CTA finds its codes and scales in a raw stage.
// Gate/up: rows 32q + l hold gate (l < 16) or up (l >= 16) of intermediate
// 16q + (l & 15); the stage holds 64 gate rows, then 64 up rows.
template <int MODE>
__device__ inline void raw_row(int r, int &code_off, int &swz, int &scale_off) {
    int br, srow;
    if (MODE == 0) {
        const int q = r >> 5, l = r & 31;
        br = 16 * q + (l & 15);
        code_off = (l < 16 ? 0 : kRawCodeBytes / 2) + br * 128;
        srow = l < 16 ? br : 64 + br;
    } else {
        br = r;
        code_off = r * 128;
        srow = r;
    }
    swz = br & 7;                 // 128-byte swizzle of the TMA box: chunk c at c ^ (row & 7)
    scale_off = kRawCodeBytes + srow * 16;
}

// Writes half `hf` (64 bytes: 32 F16 weights) of A row r in the 128B-swizzled
// layout from 16 code bytes and the two E4M3 scales of those 32 weights.
__device__ inline void store_half_row(uint8_t *a_stage, int r, int hf, uint4 c, uint32_t s2) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint8_t *row = a_stage + r * 128;
#pragma unroll
    for (int jj = 0; jj < 4; jj++) {
        const int j = 4 * hf + jj;   // 16-byte chunk of the row: weights 8j..8j+7
        const uint32_t sc = e4m3_to_f16x2_bcast(s2 >> (8 * (jj >> 1)));
        uint32_t o0, o1, o2, o3;
        e2m1x8_to_f16(w[jj], o0, o1, o2, o3);
        uint4 v = make_uint4(hmul2(o0, sc), hmul2(o1, sc), hmul2(o2, sc), hmul2(o3, sc));
        *reinterpret_cast<uint4 *>(row + ((j ^ (r & 7)) << 4)) = v;
    }
}

// Accumulator columns at or past `nvalid` belong to no pair of the tile (the MMA
// ran over the pairs rounded up to 16, and TMEM columns past that keep whatever
// an earlier tile left): zeroed, so that nothing computed from them is flagged
// or stored as a real value.
__device__ inline void zero_past(uint32_t (&v)[32], int nvalid) {
    if (nvalid < 32) {
#pragma unroll
        for (int j = 0; j < 32; j++) v[j] = j < nvalid ? v[j] : 0u;
    }
}

// Named barrier over the four epilogue warps (id 0 is __syncthreads).
__device__ inline void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// The same barrier with an AND over the 128 epilogue threads: every epilogue
// thread leaves the tile loop together.
__device__ inline bool epi_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n"
        " selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Copies a staged chunk (ncol columns of kRowsB F16 values, each column contiguous
// in shared memory) to `ncol` rows of `dst` (row stride `ld` elements), by the 128
// epilogue threads with 16-byte accesses; only the first `nrows` values of each
// column (a multiple of 8) are stored. Every shared load is issued before the
// first global store: the compiler cannot tell the two apart and would otherwise
// wait for each store before the next load.
template <int kRowsB>
__device__ inline void store_chunk(const __half *stage, __half *dst, size_t ld, int ncol, int nrows) {
    constexpr int kParts = kRowsB / 8, kPer = 32 * kParts / 128;
    const int nq = ncol * kParts, vparts = nrows / 8;
    uint4 val[kPer];
#pragma unroll
    for (int k = 0; k < kPer; k++) {
        const int q = threadIdx.x + 128 * k;
        if (q < nq) val[k] = reinterpret_cast<const uint4 *>(stage)[q];
    }
#pragma unroll
    for (int k = 0; k < kPer; k++) {
        const int q = threadIdx.x + 128 * k;
        if (q < nq && q % kParts < vparts)
            reinterpret_cast<uint4 *>(dst + (size_t)(q / kParts) * ld)[q % kParts] = val[k];
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const Params p, const __grid_constant__ CUtensorMap map_b,
                        const __grid_constant__ CUtensorMap map_a0,
                        const __grid_constant__ CUtensorMap map_a1,
                        const __grid_constant__ CUtensorMap map_y) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *a_base = smem;
    uint8_t *b_base = smem + kRing * kAStage;
    uint8_t *raw_base = b_base + kRing * kBStage;
    uint8_t *epi_stage = raw_base + kRawStages * kRawBytes;
    float *colf_s = reinterpret_cast<float *>(epi_stage + kEpiBytes);
    float *colu_s = colf_s + kBN;                 // gate/up: the up factor (see the epilogue)
    Bars *bars = reinterpret_cast<Bars *>(epi_stage + kEpiBytes + 2 * kColBytes);
    volatile int *abort = &bars->abort;
    // The small-expert kernel that follows on the stream reads nothing this grid
    // writes: it may take the SMs this grid leaves while its last tiles run.
    grid_dep_launch();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const bool leader = rank == 0;
    const int cid = (int)blockIdx.x >> 1, ncl = (int)gridDim.x >> 1;
    const Tile *tiles = MODE == 0 ? p.tiles_gu : p.tiles_dn;
    const int ntiles = p.cnt[MODE == 0 ? kCntTilesGu : kCntTilesDn];
    const int Kdim = MODE == 0 ? p.H : p.I;
    // K steps: K rounded up to a multiple of 128 (the dequant warps take steps in
    // pairs); codes past K arrive as zeros (tensor-map fill) and their scales are
    // written as zeros, so the padding adds nothing.
    const int nk = 2 * cdiv(Kdim, 2 * kBK);
    const int ntl = ntiles > cid ? cdiv(ntiles - cid, ncl) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRing; s++) {
            mbar_init(&bars->a_full[s], 17);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 8);
        }
        for (int s = 0; s < kRawStages; s++) {
            mbar_init(&bars->raw_full[s], 1 + 32);
            mbar_init(&bars->raw_empty[s], 8);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == 13) {
        tmem_alloc_pair(&bars->tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 12 && lane == 0) tma_prefetch_desc(&map_b);
    if (warp == 14 && lane == 0) {
        tma_prefetch_desc(&map_a0);
        if (MODE == 0) tma_prefetch_desc(&map_a1);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();     // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_slot;

    if (warp >= 4 && warp < 12) {
        // ------------------------------------------------ dequantise A rows
        // Thread (r, hf) converts half hf of A row r at every K step, reading the
        // codes and scales of the current raw stage from shared memory.
        const int r = (threadIdx.x - 128) & (kBM - 1), hf = (threadIdx.x - 128) >> 7;
        int code_off, swz, scale_off;
        raw_row<MODE>(r, code_off, swz, scale_off);
        Ring<kRing> ring;
        Ring<kRawStages> rr;
        uint4 s4 = make_uint4(0, 0, 0, 0);
        bool ok = true;
        // One ring stage (two 64-wide K blocks) per iteration: K is a multiple of
        // 128, so every tile has an even number of 64-wide steps; one wait, one
        // proxy fence and one arrival per stage.
        for (int tl = 0; ok && tl < ntl; tl++) {
            for (int kk = 0; kk < nk; kk += 2) {
                const int kq = kk % kRawSteps;   // 0 or 2
                const uint8_t *raw = raw_base + rr.stage * kRawBytes;
                if (kq == 0) {
                    const bool g = mbar_wait(&bars->raw_full[rr.stage], rr.phase, abort, p.status, 9);
                    if (!__all_sync(0xffffffffu, g)) {
                        ok = false;
                        break;
                    }
                    s4 = *reinterpret_cast<const uint4 *>(raw + scale_off);
                }
                const int s0 = ring.stage;
                const bool got = mbar_wait(&bars->empty[s0], ring.phase ^ 1, abort, p.status, 1);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const uint4 code0 = *reinterpret_cast<const uint4 *>(raw + code_off + (((2 * kq + hf) ^ swz) << 4));
                const uint4 code1 = *reinterpret_cast<const uint4 *>(raw + code_off + (((2 * kq + 2 + hf) ^ swz) << 4));
                const uint32_t sw0 = kq == 0 ? s4.x : s4.z, sw1 = kq == 0 ? s4.y : s4.w;
                store_half_row(a_base + s0 * kAStage, r, hf, code0, sw0 >> (16 * hf));
                store_half_row(a_base + s0 * kAStage + kSubBytes, r, hf, code1, sw1 >> (16 * hf));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(&bars->a_full[s0], 0));
                ring.next();
                if (kq + 1 == kRawSteps - 1 || kk + 2 == nk) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->raw_empty[rr.stage]);
                    rr.next();
                }
            }
        }
    } else if (warp == 14) {
        // ------------------------------------------- raw weight stages (A)
        // Per tile and 4 K steps: the codes of this CTA's 128 rows by TMA (one
        // 64-row box per gate and up plane, or one 128-row box of down), the
        // scales by 8-byte copies from all 32 lanes (a scale row's stride need
        // not be a multiple of 16 bytes, which a tensor map would require). When K
        // is not a multiple of 128 a row's scales need not be 8-byte aligned: they
        // are then copied 2 bytes at a time by plain loads, with zeros past the
        // row's end and for rows past the plane (a partial last tile of the last
        // expert).
        const int kd16 = Kdim / 16;   // scale bytes per weight row
        const bool narrow = Kdim % 128 != 0;
        const int plane_rows = MODE == 0 ? p.E * p.I : p.E * p.H;
        Ring<kRawStages> rr;
        uint32_t issued = 0, issued_phase = 0;
        bool ok = true;
        for (int tl = 0; ok && tl < ntl; tl++) {
            const Tile t = tiles[cid + tl * ncl];
            const int row0 = half_row0<MODE>(p, t, rank);
            const uint8_t *sc0 = (MODE == 0 ? p.gate_scales : p.down_scales) + (size_t)row0 * kd16;
            const uint8_t *sc1 = MODE == 0 ? p.up_scales + (size_t)row0 * kd16 : nullptr;
            for (int R = 0; R < cdiv(nk, kRawSteps); R++) {
                const bool g = mbar_wait(&bars->raw_empty[rr.stage], rr.phase ^ 1, abort, p.status, 10);
                if (!__all_sync(0xffffffffu, g)) {
                    ok = false;
                    break;
                }
                uint8_t *raw = raw_base + rr.stage * kRawBytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars->raw_full[rr.stage], kRawCodeBytes);
                    if (MODE == 0) {
                        tma_load_2d(raw, &map_a0, &bars->raw_full[rr.stage], 128 * R, row0);
                        tma_load_2d(raw + kRawCodeBytes / 2, &map_a1, &bars->raw_full[rr.stage], 128 * R, row0);
                    } else {
                        tma_load_2d(raw, &map_a0, &bars->raw_full[rr.stage], 128 * R, row0);
                    }
                    issued |= 1u << rr.stage;
                    issued_phase = (issued_phase & ~(1u << rr.stage)) | (rr.phase << rr.stage);
                }
                if (!narrow) {
                    // 128 rows x two 8-byte pieces; pieces past the row's end are
                    // skipped (their K steps are never converted), and so are rows
                    // past the plane (their codes arrive as zeros and their results
                    // are dropped)
#pragma unroll
                    for (int k = 0; k < (2 * kBM) / 32; k++) {
                        const int ci = lane + 32 * k, row = ci >> 1, off = 16 * R + 8 * (ci & 1);
                        const int prow = MODE == 0 ? row & 63 : row;
                        if (off < kd16 && row0 + prow < plane_rows) {
                            const uint8_t *src = MODE == 0 ? (row < 64 ? sc0 + (size_t)row * kd16
                                                                       : sc1 + (size_t)(row - 64) * kd16)
                                                           : sc0 + (size_t)row * kd16;
                            cp_async8(raw + kRawCodeBytes + row * 16 + 8 * (ci & 1), src + off);
                        }
                    }
                    cp_async_arrive_noinc(&bars->raw_full[rr.stage]);
                } else {
                    // 128 rows x eight 2-byte pieces, zeros where there is no scale
#pragma unroll 8
                    for (int k = 0; k < (8 * kBM) / 32; k++) {
                        const int ci = lane + 32 * k, row = ci >> 3, off = 16 * R + 2 * (ci & 7);
                        const int prow = MODE == 0 ? row & 63 : row;   // row within its plane's box
                        unsigned short v = 0;
                        if (off < kd16 && row0 + prow < plane_rows) {
                            const uint8_t *src = MODE == 0 ? (row < 64 ? sc0 : sc1) : sc0;
                            v = *reinterpret_cast<const unsigned short *>(src + (size_t)prow * kd16 + off);
                        }
                        *reinterpret_cast<unsigned short *>(raw + kRawCodeBytes + row * 16 + 2 * (ci & 7)) = v;
                    }
                    mbar_arrive(&bars->raw_full[rr.stage]);
                }
                rr.next();
            }
        }
        // Every raw stage this warp filled must have landed before exit.
        if (lane == 0)
            for (int s = 0; s < kRawStages; s++)
                if (issued & (1u << s))
                    mbar_wait_drain(&bars->raw_full[s], (issued_phase >> s) & 1, kDrainNs);
        __syncwarp();
    } else if (warp == 12) {
        // ------------------------------------------------------ TMA for B
        // This CTA's half of the tile's pair rows, in 64-row boxes; the bytes are
        // counted on the leader's a_full, whose one arrival from this warp (with the byte
        // count of both halves) the leader makes. The next tile's descriptor is
        // read one tile ahead.
        if (lane == 0) {
            Cursor cs(nk / kSub, ntiles, cid, ncl);   // steps over ring stages (128 K)
            Ring<kRing> ring;
            uint32_t issued = 0, issued_phase = 0;  // leader: stages with a load in flight
            int cur_tile = -1;
            Tile t{}, t_n{};
            if (cs.valid()) t_n = tiles[cs.tile()];
            while (cs.valid()) {
                if (cs.tile() != cur_tile) {
                    cur_tile = cs.tile();
                    t = t_n;
                    if (cur_tile + ncl < ntiles) t_n = tiles[cur_tile + ncl];
                }
                if (!mbar_wait(&bars->empty[ring.stage], ring.phase ^ 1, abort, p.status, 2)) break;
                const int half = ((t.ntok + 15) & ~15) >> 1;
                const int nbox = cdiv(half, kBBox);
                uint8_t *bs = b_base + ring.stage * kBStage;
                if (leader) {
                    mbar_arrive_expect_tx(&bars->a_full[ring.stage], kSub * 2 * nbox * kBoxBytes);
                    issued |= 1u << ring.stage;
                    issued_phase = (issued_phase & ~(1u << ring.stage)) | (ring.phase << ring.stage);
                }
                const uint32_t bar = mapa_shared(&bars->a_full[ring.stage], 0);
                for (int sb = 0; sb < kSub; sb++)
                    for (int b = 0; b < nbox; b++)
                        tma_load_2d_pair(bs + sb * kSubBytes + b * kBoxBytes, &map_b, bar,
                                         (kSub * cs.kk + sb) * kBK, t.pos0 + rank * half + b * kBBox);
                ring.next();
                cs.next();
            }
            // The leader's last load of every stage must have landed before exit.
            for (int s = 0; s < kRing; s++)
                if (issued & (1u << s))
                    mbar_wait_drain(&bars->a_full[s], (issued_phase >> s) & 1, kDrainNs);
        }
    } else if (warp == 13) {
        // ---------------------------------------------- pair MMA issue (leader)
        if (leader && lane == 0) {
            // This one thread paces the tile (the operands are almost always ready
            // when it gets to them), so its K step is kept short: one barrier per
            // stage (A arrivals and B bytes together), the next stage's barrier
            // tested without blocking while this stage's MMAs go out, each stage's
            // descriptors computed once (a k16 step adds 32 bytes, i.e. 2, to the
            // address field; the second 64-wide block of a stage 16 KB), and
            // stages of 128 K: eight MMAs per wait, test and commit.
            Ring<kRing> ring;
            uint32_t acc_phase = 0;     // bit b: parity of accumulator b's next use
            bool ok = true;
            uint64_t adesc[kRing], bdesc[kRing];
#pragma unroll
            for (int st = 0; st < kRing; st++) {
                adesc[st] = smem_desc_sw128(smem_u32(a_base + st * kAStage));
                bdesc[st] = smem_desc_sw128(smem_u32(b_base + st * kBStage));
            }
            bool ready = false;   // the current stage's barrier already seen complete
            for (int tl = 0; ok && tl < ntl; tl++) {
                const Tile t = tiles[cid + tl * ncl];
                const int buf = tl & 1;
                const int nmma = (t.ntok + 15) & ~15;
                const uint32_t idesc = idesc_f16(2 * kBM, nmma);
                if (!mbar_wait(&bars->acc_empty[buf], ((acc_phase >> buf) & 1) ^ 1, abort, p.status, 4))
                    break;
                acc_phase ^= 1u << buf;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * kBN;
                // one ring stage (two 64-wide K blocks, eight MMAs) per iteration
                for (int ks = 0; ks < nk / kSub; ks++) {
                    if (!ready && !mbar_wait(&bars->a_full[ring.stage], ring.phase, abort, p.status, 5)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    Ring<kRing> nx = ring;
                    nx.next();
                    ready = mbar_test(&bars->a_full[nx.stage], nx.phase);
                    uint64_t ad = adesc[0], bd = bdesc[0];
#pragma unroll
                    for (int st = 1; st < kRing; st++)
                        if (ring.stage == st) {
                            ad = adesc[st];
                            bd = bdesc[st];
                        }
#pragma unroll
                    for (int sb = 0; sb < kSub; sb++)
#pragma unroll
                        for (int k16 = 0; k16 < kBK / 16; k16++)
                            tc_mma_f16_pair(d_tmem, ad + sb * (kSubBytes >> 4) + 2 * k16,
                                            bd + sb * (kSubBytes >> 4) + 2 * k16, idesc, (ks | sb | k16) != 0);
                    tc_commit_pair_mc(&bars->empty[ring.stage], kBothCtas);
                    ring = nx;
                }
                if (ok) tc_commit_pair_mc(&bars->acc_full[buf], kBothCtas);
            }
            // Drain: every MMA this thread issued completes before TMEM is freed.
            tc_commit_pair(&bars->drain);
            mbar_wait_drain(&bars->drain, 0, kDrainNs);
        }
    } else {
        // -------------------------------------------------------- epilogue
        // Per tile: the tile's per-column factors (activation scale, or routing
        // weight x s_d) are loaded before the accumulator wait and parked in
        // shared memory; each 32-column chunk is staged in shared memory (two
        // buffers, one named barrier per chunk) and written with coalesced 16-byte
        // stores.
        constexpr int kChunks = kBN / 32;
        uint32_t acc_phase = 0;
        for (int tl = 0; tl < ntl; tl++) {
            const Tile t = tiles[cid + tl * ncl];
            const int buf = tl & 1;
            const int e = t.expert;
            // gate/up: x's staging factor for g, and for u that factor times 2^hexp
            // of the pair's token (h is stored relative to it; the combine undoes
            // it); down: routing weight x s_d
            const float *colf = MODE == 0 ? p.ps : p.pw;
            const float cscale = MODE == 0 ? 1.0f : p.down_global[e];
            float cf[kBN / 128], cu[kBN / 128];
#pragma unroll
            for (int c = 0; c < kBN / 128; c++) {
                const int col = 128 * c + threadIdx.x;
                cf[c] = col < t.ntok ? colf[t.pos0 + col] * cscale : 0.0f;
                if (MODE == 0) cu[c] = col < t.ntok ? cf[c] * p.ph[t.pos0 + col] : 0.0f;
            }
            const bool got = mbar_wait(&bars->acc_full[buf], (acc_phase >> buf) & 1, abort, p.status, 8);
            // The AND-barrier also orders every read of colf_s for the previous
            // tile before the writes below.
            if (!epi_all(got)) break;
#pragma unroll
            for (int c = 0; c < kBN / 128; c++) {
                colf_s[128 * c + threadIdx.x] = cf[c];
                if (MODE == 0) colu_s[128 * c + threadIdx.x] = cu[c];
            }
            epi_sync();
            acc_phase ^= 1u << buf;
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * kBN + ((uint32_t)(warp * 32) << 16);
            if (MODE == 0) {
                // SwiGLU; h staged as [32 columns][64 intermediates] F16 (each column
                // is 128 contiguous bytes of h).
                const float sg = p.gate_global[e], su = p.up_global[e];
                const int il = 16 * warp + (lane & 15);
                const bool is_gate = lane < 16;
                const int i0 = t.m0 + kGuCta * rank;
                // intermediates of this half inside I (a partial last tile when I is
                // not a multiple of 128 reads the next expert's rows; dropped)
                const int ni = max(0, min(kGuCta, p.I - i0));
                const bool row_ok = il < ni;
                bool fin = true;
#pragma unroll 1
                for (int c = 0; c < kChunks; c++) {
                    if (32 * c >= t.ntok) break;
                    __half *hs = reinterpret_cast<__half *>(epi_stage) + (c & 1) * (32 * kGuCta);
                    // This lane's 16 column factors, in registers before the first
                    // staging store (shared loads after it would wait for it).
                    const int cj0 = is_gate ? 0 : 16;
                    float xs[16], xu[16];
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        const float4 f = reinterpret_cast<const float4 *>(colf_s + 32 * c + cj0)[k];
                        xs[4 * k] = f.x; xs[4 * k + 1] = f.y; xs[4 * k + 2] = f.z; xs[4 * k + 3] = f.w;
                        const float4 g = reinterpret_cast<const float4 *>(colu_s + 32 * c + cj0)[k];
                        xu[4 * k] = g.x; xu[4 * k + 1] = g.y; xu[4 * k + 2] = g.z; xu[4 * k + 3] = g.w;
                    }
                    uint32_t v[32];
                    tmem_ld32(tbase + 32 * c, v);
                    tmem_ld_wait();
                    zero_past(v, t.ntok - 32 * c);
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float mine_lo = __uint_as_float(v[j]);
                        const float mine_hi = __uint_as_float(v[16 + j]);
                        const float send = is_gate ? mine_hi : mine_lo;
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                        const float gacc = is_gate ? mine_lo : recv;
                        const float uacc = is_gate ? recv : mine_hi;
                        const float gv = gacc * sg * xs[j], uv = uacc * su * xu[j];
                        const float hf = silu(gv) * uv;
                        fin &= fits_f16(hf) || !row_ok;
                        hs[(cj0 + j) * kGuCta + il] = __float2half_rn(hf);
                    }
                    epi_sync();
                    if (ni > 0)
                        store_chunk<kGuCta>(hs, p.h + (size_t)(t.pos0 + 32 * c) * p.I + i0, p.I,
                                            min(32, t.ntok - 32 * c), ni);
                }
                // h is stored in F16: a value past its range is reported, not hidden
                if (!fin) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfH | e);
            } else {
                // y * s_d * w staged as [32 columns][128 hidden rows] F16, written into
                // the pair's row of yp; the combine kernel sums each token's K rows in
                // a fixed order.
                const int r = 32 * warp + lane;
                const int m = t.m0 + kBM * rank;
                const int nr = min(kBM, p.H - m);   // rows of this half inside H
                const bool row_ok = r < nr;
                bool fin = true;
                if (m < p.H) {
#pragma unroll 1
                    for (int c = 0; c < kChunks; c++) {
                        if (32 * c >= t.ntok) break;
                        __half *ys = reinterpret_cast<__half *>(epi_stage) + (c & 1) * (32 * kBM);
                        // A whole chunk (32 pairs, 128 rows inside H) leaves by one bulk
                        // tensor store from this staging buffer; the store issued from it
                        // two chunks ago must have finished reading it first.
                        const bool whole = t.ntok - 32 * c >= 32 && nr == kBM;
                        if (threadIdx.x == 0) bulk_wait_read_1();
                        epi_sync();
                        // The chunk's 32 column factors in registers before the first
                        // staging store.
                        float cf[32];
#pragma unroll
                        for (int k = 0; k < 8; k++) {
                            const float4 f = reinterpret_cast<const float4 *>(colf_s + 32 * c)[k];
                            cf[4 * k] = f.x; cf[4 * k + 1] = f.y; cf[4 * k + 2] = f.z; cf[4 * k + 3] = f.w;
                        }
                        uint32_t v[32];
                        tmem_ld32(tbase + 32 * c, v);
                        tmem_ld_wait();
                        zero_past(v, t.ntok - 32 * c);
#pragma unroll
                        for (int j = 0; j < 32; j++) {
                            const float yf = __uint_as_float(v[j]) * cf[j];
                            fin &= fits_f16(yf) || !row_ok;
                            ys[j * kBM + r] = __float2half_rn(yf);
                        }
                        if (whole) {
                            fence_proxy_async_smem();   // the staging writes, before the bulk copy reads them
                            epi_sync();
                            if (threadIdx.x == 0) {
                                tma_store_2d(&map_y, ys, m, t.pos0 + 32 * c);
                                bulk_commit();
                            }
                        } else {
                            epi_sync();
                            store_chunk<kBM>(ys, p.xh + (size_t)(t.pos0 + 32 * c) * p.H + m, p.H,
                                             min(32, t.ntok - 32 * c), nr);
                        }
                    }
                }
                // the per-pair rows w * s_d * y are stored in F16 (see above)
                if (!fin) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, kNfY | e);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(&bars->acc_empty[buf], 0));
        }
        // every bulk store of the down rows complete before the CTA ends
        if (threadIdx.x == 0) bulk_wait_all();
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort) {
        // After a give-up, copies this CTA started may still be landing in its
        // shared memory (the peer's loads are counted on the leader's barrier).
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < kSettleNs) __nanosleep(1000);
    }
    __syncthreads();
    cluster_sync_all();     // no pair MMA, copy or remote arrive touches either CTA past here
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

static cudaLaunchConfig_t gemm_config(int nclusters, cudaStream_t s, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * nclusters);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes();
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

cudaError_t prefill_init(int *max_clusters) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<0>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem_bytes());
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = gemm_config(1, 0, attr);
    int n0 = 0, n1 = 0;
    e = cudaOccupancyMaxActiveClusters(&n0, grouped_gemm_kernel<0>, &cfg);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveClusters(&n1, grouped_gemm_kernel<1>, &cfg);
    if (e != cudaSuccess) return e;
    *max_clusters = n0 < n1 ? n0 : n1;
    return *max_clusters > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t launch_prefill_gemm(int mode, const Params &p, const CUtensorMap &map_b,
                                const CodeMaps &codes, const CUtensorMap &map_y, int max_clusters,
                                cudaStream_t s) {
    const int maxt = mode == 0 ? p.max_tiles_gu : p.max_tiles_dn;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = gemm_config(max(1, min(max_clusters, maxt)), s, attr);
    return mode == 0 ? cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<0>, p, map_b, codes.gate, codes.up, map_y)
                     : cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<1>, p, map_b, codes.down, codes.down, map_y);
}

}  // namespace nvmoe
