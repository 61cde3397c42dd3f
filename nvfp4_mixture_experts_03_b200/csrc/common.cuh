// Device helpers shared by the layer's kernels (sm_100a only): status latching,
// bounded mbarrier waits, TMA loads, tcgen05 (TMEM alloc / MMA / commit / load),
// NVFP4 conversions, and the workspace / launch-parameter layout.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "nvfp4_moe.h"
#include "nvfp4_moe_test.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace nvmoe {

// ---------------------------------------------------------------- constants
constexpr int kChunkTokens = 64;       // tokens per routing CTA (two 32-bit token masks)
constexpr int kBN = 256;               // max tokens per grouped-GEMM tile (MMA N)
constexpr int kBK = 64;                // K elements per pipeline stage (one 128B swizzle row)
// Grouped-GEMM tiles are computed by a pair of CTAs (one cluster, one M = 256 MMA):
constexpr int kGuRows = 128;           // intermediates per gate/up tile (64 per CTA: 64 gate + 64 up rows)
constexpr int kDnRows = 256;           // hidden rows per down tile (128 per CTA; the last may be half)

// Device status block layout (int32 words, 256 bytes): the latched error and its
// detail.
enum : int { kStatusCode = 0, kStatusDetail = 1, kStatusWords = 64 };

// Per-call routing/tile counters kept in the workspace (int32 words).
// kCntSmallQ, +1: the small-expert kernels' item queues (gate/up, down).
enum : int { kCntTilesGu = 0, kCntTilesDn = 1, kCntUniq = 2, kCntSmall = 3, kCntSmallQ = 4, kCntWords = 64 };
// Experts with at most this many pairs skip the grouped-GEMM tiles and are
// streamed through mma.sync instead (two 8-token halves of one m16n8k16 pass).
constexpr int kSmallTok = 16;
// Decode state (per handle, int32 counters): kDsArrive: CTAs at the grid barrier
// (zero between launches); kDsGen: barrier generation (counts launches; any
// value is valid, so the state may be cleared at any time between launches).
enum : int { kDsArrive = 0, kDsGen = 1, kDsInts = 64 };
inline size_t decode_state_bytes() { return (size_t)kDsInts * 4; }

struct Tile {  // one grouped-GEMM tile
    int32_t expert;   // expert id
    int32_t m0;       // first output row (gate/up: intermediate index; down: hidden index)
    int32_t pos0;     // first pair position (rows of the permuted activations / h)
    int32_t ntok;     // valid pairs in this tile (1..kBN)
};

// Everything a forward call's kernels read, passed by value.
struct Params {
    int32_t T, E, H, I, K;
    int32_t act_type;          // nvfp4_moe_act, plus kActF32 below
    int32_t out_add;           // 1: out += layer(x)
    const void *act;
    const float *act_scale;
    const float *logits;       // may be null
    const uint16_t *router_w;  // [E][H] bf16 router projection, or null
    float *rlogits;            // [T][E] logits the router projection writes
    const int32_t *in_ids;     // precomputed routing when logits == null
    const float *in_w;
    float *out;
    // weights
    const uint8_t *gate_codes, *up_codes, *gate_scales, *up_scales;
    const float *gate_global, *up_global;
    const uint8_t *down_codes, *down_scales;
    const float *down_global;
    // workspace regions
    int32_t *cnt;              // kCntWords counters
    int32_t *ids;              // [P]
    float *wts;                // [P]
    int32_t *hist;             // [E][nch]
    int32_t *cbase;            // [E][nch]
    int32_t *counts;           // [E]
    int32_t *offsets;          // [E+1]
    int32_t *perm;             // [P] pair index at each position
    int32_t *inv;              // [P] position of each pair
    int32_t *ptok;             // [P] token at each position
    float *pw;                 // [P] routing weight at each position
    float *ps;                 // [P] activation scale at each position (prefill)
    float *xscale;             // [T] activation scale per token
    float *ph;                 // [P] prefill: 2^hexp of the pair's token at each position
    float *phinv;              // [T] prefill: 2^-hexp per token
    Tile *tiles_gu, *tiles_dn;
    int32_t *small_e;          // [E] prefill: experts with 1..small_tok pairs, ascending
    int32_t small_tok;         // prefill: pair count up to which an expert is small (0: none)
    __half *xh;                // prefill: [P][H] F16 activations per pair position, then the
                               // down projection's w * s_d * y per pair (F16)
    __half *h;                 // [P][I]
    int32_t *status;           // device status block
    // optional debug copies
    int32_t *dbg_ids;
    float *dbg_w;
    int32_t *dbg_counts, *dbg_offsets, *dbg_perm;
    int32_t nch;               // routing chunks
    int32_t max_tiles_gu, max_tiles_dn;
    int32_t *dstate;           // decode: counters (kDs*), zero between launches
    int32_t dec_union;         // decode: bytes of the phase-shared dynamic shared memory
    int32_t test_flags;        // NVFP4_MOE_TEST_* (test hooks; 0 in production)
};

constexpr int kActF32 = 2;     // internal: act is FP32, rounded to BF16 first

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------ status
__device__ inline void latch_status(int32_t *status, int code, int detail) {
    if (atomicCAS(&status[kStatusCode], 0, code) == 0) status[kStatusDetail] = detail;
}
// Detail words of NVFP4_MOE_ERR_NONFINITE when a computed value is not finite
// (routing reports the token index instead, always < 2^20): which stored
// intermediate, ORed with the expert id.
enum : int { kNfH = 1 << 20, kNfY = 2 << 20, kNfOut = 3 << 20 };
// An FP32 value stays finite when rounded to F16 iff its magnitude is below
// 65520 (65504 plus half an F16 ulp rounds to inf); NaN fails the compare.
__device__ inline bool fits_f16(float x) { return fabsf(x) < 65520.0f; }

// --------------------------------------------------------------- utilities
__device__ inline uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Programmatic dependent launch: wait for the grid this one depends on (its
// writes visible); let the grid that depends on this one start launching.
__device__ inline void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

__device__ inline uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ inline void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ inline void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ inline void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}
template <bool kCluster = false>
__device__ inline bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    if (kCluster)   // arrivals may come from the other CTA of the cluster
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
    else
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
    return ok != 0;
}
// Bounded wait: gives up after `limit_ns` of wall time (or when *abort is set by
// another thread), latching NVFP4_MOE_ERR_TIMEOUT. Returns false on give-up.
template <bool kCluster = false>
__device__ inline bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                 int32_t *status, int where, uint64_t limit_ns = 2000000000ull) {
    if (mbar_try_wait<kCluster>(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait<kCluster>(bar, parity)) return true;
        if ((++spins & 63) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > limit_ns) {
                *abort = 1;
                latch_status(status, NVFP4_MOE_ERR_TIMEOUT, where);
                return false;
            }
        }
    }
}

// Bounded wait used when draining after a give-up: ignores the abort flag, never
// latches a status, returns false after `limit_ns`.
__device__ inline bool mbar_wait_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > limit_ns) return false;
    return true;
}

// ------------------------------------------------- clusters of two CTAs
__device__ inline uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster (warps must be converged).
__device__ inline void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ inline uint32_t mapa_shared(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrive on an mbarrier of any CTA of the cluster (default .release.cta
// semantics: a cluster-scope release would also wait for this thread's
// outstanding global loads, i.e. drain the dequant prefetch at every arrival).
__device__ inline void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ inline void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ inline void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// --------------------------------------------------------------------- TMA
__device__ inline void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x,
                                   int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
// Pair form: the box lands in this CTA's shared memory and its bytes are counted
// on the mbarrier at `bar_cluster` (a shared::cluster address, here the leader
// CTA's). No multicast.
__device__ inline void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster,
                                        int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}
// 8-byte asynchronous copy global -> shared (both 8-byte aligned).
__device__ inline void cp_async8(void *dst_smem, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst_smem)), "l"(src)
                 : "memory");
}
// Arrives on `bar` when every cp.async this thread issued so far has landed; the
// arrival is counted in the barrier's initial count (.noinc).
__device__ inline void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ inline void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// ----------------------------------------------------------------- tcgen05
// Pair forms (cta_group::2): one warp with the same warp index in each CTA of the
// pair issues alloc / relinquish / dealloc; the same columns are taken in both.
__device__ inline void tmem_alloc_pair(uint32_t *slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot_smem)),
                 "r"(ncols));
}
__device__ inline void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}
__device__ inline void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ inline void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ inline void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Pair MMA (issued by the leader CTA only): M = 256 rows, the first 128 from the
// leader's A tile and TMEM, the next 128 from the peer's; B's first N/2 rows from
// the leader's shared memory and the other N/2 from the peer's (same offsets).
__device__ inline void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrives on the mbarrier at the same offset in every CTA of `cta_mask` once the
// pair MMAs issued so far by this thread have completed.
__device__ inline void tc_commit_pair_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
__device__ inline void tc_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: this thread gets its lane's 32 columns.
__device__ inline void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ inline void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand tile in the 128-byte swizzle
// layout (rows of 128 B, 8-row groups 1024 B apart). Start address in 16-B units.
__device__ inline uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);            // start address
    d |= (uint64_t)1 << 16;                             // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;                   // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                             // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                             // layout: 128-byte swizzle
    return d;
}
// Instruction descriptor, kind::f16: F16 x F16 -> F32, both K-major, M x N.
__host__ __device__ inline uint32_t idesc_f16(int M, int N) {
    return (1u << 4)                      // D format F32
           | (0u << 7) | (0u << 10)       // A, B format F16
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// ------------------------------------------------------- NVFP4 conversions
// Four E2M1 code bytes -> four f16x2 (low nibble -> low half: element 2c first).
__device__ inline void e2m1x8_to_f16(uint32_t c, uint32_t &o0, uint32_t &o1, uint32_t &o2,
                                     uint32_t &o3) {
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
        " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
        : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
        : "r"(c));
}
// One E4M3 scale byte -> f16x2 with the scale in both halves (exact: E4M3 is a
// subset of F16).
__device__ inline uint32_t e4m3_to_f16x2_bcast(uint32_t s) {
    uint32_t o;
    const uint16_t two = (uint16_t)((s & 0xFF) | ((s & 0xFF) << 8));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(o) : "h"(two));
    return o;
}
__device__ inline uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// ----------------------------------------------------------------- mma.sync
// D[16x8] += A[16x16] (row) x B[16x8] (col), F16 inputs, F32 accumulate.
__device__ inline void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                 uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// z * sigmoid(z) with the fast exponential and divide intrinsics (relative error
// a few FP32 ulps; z -> -inf gives exp = inf and a zero quotient).
__device__ inline float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Per-token power-of-two factor 2^k with amax * 2^k in [2^14, 2^15): every BF16
// value within 2^28 of the token's amax is exact in F16 after the shift.
__device__ inline int pow2_shift_for(float amax) {
    if (!(amax > 0.0f) || !isfinite(amax)) return 0;
    int e;
    frexpf(amax, &e);           // amax = m * 2^e, m in [0.5, 1)
    int k = 15 - e;             // amax * 2^k in [2^14, 2^15)
    return k < -120 ? -120 : (k > 120 ? 120 : k);   // keep 2^-k a normal FP32
}

// Power-of-two exponent by which a token's h values are stored (h * 2^e; also
// the grouped-GEMM path's per-pair down rows, which are built from h): 0 while
// the token's activation amax stays below 256, else -2 (m - 8) for an amax in
// [2^(m-1), 2^m), so that h, which grows with the square of the activations,
// keeps within F16's range. Exact (a power of two), undone in FP32.
__device__ inline int h_exp_for(float amax) {
    if (!(amax >= 256.0f) || !isfinite(amax)) return 0;
    int m;
    frexpf(amax, &m);           // amax in [2^(m-1), 2^m), m >= 9
    const int e = -2 * (m - 8);
    return e < -100 ? -100 : e;
}

// ------------------------------------------------------------ kernel decls
void launch_route_large(const Params &p, cudaStream_t s);
void launch_prep_prefill(const Params &p, cudaStream_t s);
void launch_combine(const Params &p, cudaStream_t s);   // prefill: per-token sum of the K pair rows
// prefill, experts with <= small_tok pairs: mode 0 gate/up + SwiGLU, mode 1 down
cudaError_t launch_small(int mode, const Params &p, cudaStream_t s);
cudaError_t small_init();
bool small_fits(int H, int I);   // the small-expert kernels' shared memory fits
cudaError_t launch_decode(const Params &p, cudaStream_t s);   // the whole T <= 8 layer
// One layer's weight planes, for a decode stack.
struct DecLayerPtrs {
    const uint8_t *gate_codes, *up_codes, *gate_scales, *up_scales;
    const float *gate_global, *up_global;
    const uint8_t *down_codes, *down_scales;
    const float *down_global;
};
// n decode layers in one launch over the FP32 residual stream
cudaError_t launch_decode_stack(const Params &p, const DecLayerPtrs *layers, int n, const float *logits,
                                cudaStream_t s);
int decode_grid();                                 // CTAs of the decode kernel (one per SM)
constexpr int kDecWarpsPerCta = 16;                // warps of a decode CTA
// Whether the decode kernel's shared-memory plan holds layers of these dims (else
// small batches take the grouped-GEMM path).
bool decode_fits(int H, int I, int K, int E);
size_t decode_union_bytes(int T, int K, int H, int I);
// mode 0: gate/up + SwiGLU, map_b = F16 activations [P][H]; mode 1: down, map_b =
// h [P][I]; both 64 x 64 boxes
// Tensor maps of the packed E2M1 code planes (bytes; 128-byte x 64-row boxes for
// gate and up, 128-row boxes for down; 128-byte swizzle).
struct CodeMaps {
    CUtensorMap gate, up, down;
};
// Clusters of two CTAs, at most `max_clusters` of them (persistent).
// map_y: the per-pair down rows (xh) as a bulk-store target, boxes of 32 pairs x
// 128 hidden rows (used by mode 1)
cudaError_t launch_prefill_gemm(int mode, const Params &p, const CUtensorMap &map_b,
                                const CodeMaps &codes, const CUtensorMap &map_y, int max_clusters,
                                cudaStream_t s);
// Per device: opt the GEMM kernels into their shared memory; *max_clusters = how
// many CTA pairs of either GEMM can be resident at once.
cudaError_t prefill_init(int *max_clusters);
cudaError_t decode_init();    // per device: opt the decode kernels into their shared memory
cudaError_t router_init();    // per device: opt the router GEMM into its shared memory
cudaError_t launch_router(const Params &p, cudaStream_t s);   // logits = x . W_r^T into p.rlogits

}  // namespace nvmoe
