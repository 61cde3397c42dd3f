// Small experts of the grouped-GEMM path: experts that receive at most
// kSmallTok (token, slot) pairs in one call.
//
// The pages run every expert group of a prefill chunk as one grouped launch
// ("Strata NVFP4" README, "How it differs from upstream Strata"); their
// MoE layers route by top-k over many experts, so a skewed batch leaves a long
// tail of experts with a handful of tokens. A tensor-core tile of the grouped
// GEMM costs nearly the same for 4 tokens as for 256 (the time of a K step
// hardly depends on the tile's N), so those experts are taken out of the tile
// lists and streamed here instead, like the decode layer does: each
// weight byte is read once into registers, decoded exactly to F16 and fed to
// mma.sync m16n8k16 with the expert's pairs as N (two 8-pair halves sharing
// each decoded weight fragment), FP32 accumulation.
//
// Work: the list of small experts (ascending, built with the tile lists) times
// S pieces per expert (S chosen on the device from the list's length and the
// grid, the same in every CTA) gives the items, which the CTAs take from a
// queue (one atomic per item). Each kernel is launched as a programmatic
// dependent of the tile kernel before it, which lets it start at once: its
// CTAs take the SMs the tile kernel's CTAs leave as they finish, and a CTA that
// starts late finds fewer items left. For each item the CTA stages the expert's
// pair rows (activations for gate/up, h for down) in shared memory with a zero
// row for absent pairs, and its 16 warps split the item's granules (gate/up: 8
// intermediates, gate and up rows; down: 16 hidden rows) in contiguous ranges,
// every granule whole in one warp, so each output is summed in a fixed order
// and written once, whichever CTA takes the item.
//
// Outputs match the tile kernels': gate/up stores h = silu(g) * u (F16, times
// the token's 2^hexp) at the pair's row of h; down stores y * s_d * w (F16) at
// the pair's row of the per-pair buffer that the combine kernel sums.
//
// Fragment mapping: a weight row is read in chunks of NR 128-wide K rounds.
// Thread (g = lane/4, q = lane%4) holds rows g and g+8 (the m16n8k16 A rows)
// and, in each chunk, the q-th quarter of it: 16 NR contiguous code bytes and
// 2 NR contiguous scale bytes per row (one vector load of the scales). Its
// round j of the chunk covers 32 of those K, and mma step s of the round uses
// 4 of them for the logical K {2q, 2q+1, 2q+8, 2q+9}; the staged pair rows are
// read with the same permutation, so every dot product is the plain one.
// Staged rows: stride (chunks * 128 NR + 8) F16, and inside each chunk the
// 16-byte piece u is stored at u ^ 2q (q its quarter): the eight lanes of a
// quarter warp (two rows, four q) read eight different 16-byte bank groups.
#include "common.cuh"
#include "stream_common.cuh"

namespace nvmoe {

constexpr int kSeWarps = 16;
constexpr int kSeThreads = kSeWarps * 32;
constexpr int kSeGuRounds = 2;   // gate/up: K rounds per chunk (256 K)
constexpr int kSeDnRounds = 2;   // down: K rounds per chunk (256 K)
constexpr int kSeMaxPieces = 64;

// Chunks of NR rounds per row of length K (the last one zero-padded).
__host__ __device__ inline int se_chunks(int K, int NR) { return cdiv(K, 128 * NR); }
// Row stride (F16 elements) of staged rows of length K.
__host__ __device__ inline int se_ld(int K, int NR) { return se_chunks(K, NR) * 128 * NR + 8; }
// Dynamic shared memory: kSmallTok staged rows, the zero row, and two epilogue
// factors per pair.
__host__ __device__ inline size_t se_smem(int K, int NR) {
    return (size_t)(kSmallTok + 1) * se_ld(K, NR) * 2 + 2 * kSmallTok * sizeof(float);
}
// Position in a staged row of element k (a multiple of 8: one 16-byte piece).
template <int NR>
__device__ inline int se_pos(int k) {
    const int c = k / (128 * NR), u = (k % (128 * NR)) / 8, q = u / (4 * NR);
    return c * 128 * NR + 8 * (u ^ (2 * q));
}

// Weights of one warp's chunk: this thread's quarter of rows g and g+8.
template <int NR>
struct SeBuf {
    uint4 ca[NR], cb[NR];           // 16 code bytes per round
    uint32_t sa[NR / 2], sb[NR / 2];  // two scale bytes per round
};

// Loads of chunk c of two weight rows (row a: codes `ac`, scales `as`; row b:
// `bc`, `bs`; kb code bytes per row). `v32`: the code rows allow aligned 32-byte
// loads; `vec`: the scale rows allow one aligned 2 NR-byte load. Pieces past the
// row's end are zero, with zero scales.
template <int NR>
__device__ inline void se_issue(int c, const uint8_t *ac, const uint8_t *bc, const uint8_t *as,
                                const uint8_t *bs, int kb, bool v32, bool vec, bool full, int q, SeBuf<NR> &b) {
    const int c0 = 64 * NR * c + 16 * NR * q;   // first code byte of this quarter
    const int s0 = 8 * NR * c + 2 * NR * q;     // first scale byte
    if (NR == 2 && full) {
        // every chunk whole, 32-byte code and 4-byte scale loads allowed: all loads
        // unconditional, each landing straight in its buffer register
        ldg_stream32(ac + c0, b.ca[0], b.ca[NR - 1]);
        ldg_stream32(bc + c0, b.cb[0], b.cb[NR - 1]);
        b.sa[0] = __ldg(reinterpret_cast<const uint32_t *>(as + s0));
        b.sb[0] = __ldg(reinterpret_cast<const uint32_t *>(bs + s0));
        return;
    }
    if (c0 + 16 * NR <= kb) {
        if (NR == 2 && v32) {
            ldg_stream32(ac + c0, b.ca[0], b.ca[NR - 1]);
            ldg_stream32(bc + c0, b.cb[0], b.cb[NR - 1]);
        } else {
#pragma unroll
            for (int j = 0; j < NR; j++) {
                b.ca[j] = ldg_stream(ac + c0 + 16 * j);
                b.cb[j] = ldg_stream(bc + c0 + 16 * j);
            }
        }
        if (vec) {
            if (NR == 4) {
                const uint2 va = __ldg(reinterpret_cast<const uint2 *>(as + s0));
                const uint2 vb = __ldg(reinterpret_cast<const uint2 *>(bs + s0));
                b.sa[0] = va.x;
                b.sb[0] = vb.x;
                b.sa[NR / 2 - 1] = va.y;
                b.sb[NR / 2 - 1] = vb.y;
            } else {
#pragma unroll
                for (int i = 0; i < NR / 2; i++) {
                    b.sa[i] = __ldg(reinterpret_cast<const uint32_t *>(as + s0) + i);
                    b.sb[i] = __ldg(reinterpret_cast<const uint32_t *>(bs + s0) + i);
                }
            }
            return;
        }
    }
#pragma unroll
    for (int i = 0; i < NR / 2; i++) b.sa[i] = b.sb[i] = 0;
#pragma unroll
    for (int j = 0; j < NR; j++) {
        if (c0 + 16 * j < kb) {
            if (c0 + 16 * NR > kb) {   // (already loaded when the whole quarter is inside)
                b.ca[j] = ldg_stream(ac + c0 + 16 * j);
                b.cb[j] = ldg_stream(bc + c0 + 16 * j);
            }
            const uint32_t sa = __ldg(reinterpret_cast<const unsigned short *>(as + s0 + 2 * j));
            const uint32_t sb = __ldg(reinterpret_cast<const unsigned short *>(bs + s0 + 2 * j));
            b.sa[j / 2] |= sa << (16 * (j & 1));
            b.sb[j / 2] |= sb << (16 * (j & 1));
        } else {
            b.ca[j] = b.cb[j] = make_uint4(0, 0, 0, 0);
        }
    }
}

// Round j of a chunk (eight mma steps) for both 8-pair halves: A rows g (codes
// ca, scale bytes sa) and g+8 (cb, sb); B from the staged rows at x0 (pairs
// 0..7) and x1 (pairs 8..15), offset to the chunk and this thread's quarter;
// code word w pairs with the 16 bytes at piece (4 j + w) ^ 2q.
// e2m1x8_to_f16 and hmul2 of common.cuh, issued in program order (volatile), so
// that the decode of a code word stays next to the mma steps that use it
// instead of being hoisted (which runs out of registers).
__device__ inline void se_e2m1x8(uint32_t c, uint32_t &o0, uint32_t &o1, uint32_t &o2, uint32_t &o3) {
    asm volatile("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
                 " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
                 " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
                 : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
                 : "r"(c));
}
__device__ inline uint32_t se_hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm volatile("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ inline uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
// (x0, x1: shared-memory byte addresses)
__device__ inline void se_round(float (&acc0)[4], float (&acc1)[4], const uint4 &ca, const uint4 &cb,
                                uint32_t sa, uint32_t sb, uint32_t x0, uint32_t x1, int j, int q2) {
    const uint32_t sa0 = e4m3_to_f16x2_bcast(sa & 0xFF), sa1 = e4m3_to_f16x2_bcast((sa >> 8) & 0xFF);
    const uint32_t sb0 = e4m3_to_f16x2_bcast(sb & 0xFF), sb1 = e4m3_to_f16x2_bcast((sb >> 8) & 0xFF);
    const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w}, wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t off = 16 * ((4 * j + w) ^ q2);
        const uint4 v0 = lds128(x0 + off);
        const uint4 v1 = lds128(x1 + off);
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        se_e2m1x8(wa[w], a0, a1, a2, a3);
        se_e2m1x8(wb[w], b0, b1, b2, b3);
        const uint32_t s_a = w < 2 ? sa0 : sa1, s_b = w < 2 ? sb0 : sb1;
        const uint32_t f0 = se_hmul2(a0, s_a), f1 = se_hmul2(b0, s_b), f2 = se_hmul2(a1, s_a), f3 = se_hmul2(b1, s_b);
        const uint32_t f4 = se_hmul2(a2, s_a), f5 = se_hmul2(b2, s_b), f6 = se_hmul2(a3, s_a), f7 = se_hmul2(b3, s_b);
        mma_16816(acc0, f0, f1, f2, f3, v0.x, v0.y);
        mma_16816(acc1, f0, f1, f2, f3, v1.x, v1.y);
        mma_16816(acc0, f4, f5, f6, f7, v0.z, v0.w);
        mma_16816(acc1, f4, f5, f6, f7, v1.z, v1.w);
    }
}

// Pieces per expert for nse experts of `units` granules on G CTAs: about two
// items per CTA (a CTA that starts late, or whose items run long, leaves the
// rest to the others), at most one piece per 16 granules (a granule for every
// warp) and at least one.
__device__ inline int se_pieces(int nse, int units, int G) {
    if (nse <= 0) return 1;
    const int want = cdiv(2 * G, nse), most = max(1, units / kSeWarps);
    return max(1, min(min(want, most), kSeMaxPieces));
}

// Copies the n pair rows (K F16 each, row stride K in global, se_ld here, pieces
// placed by se_pos) from `src` into xs with cp.async; the padding columns and
// the zero row were cleared once at the start.
template <int NR>
__device__ inline void se_stage(__half *xs, const __half *src, int n, int K) {
    const int ld = se_ld(K, NR), k8 = K / 8;
    for (int c = threadIdx.x; c < n * k8; c += blockDim.x) {
        const int r = c / k8, k = 8 * (c - r * k8);
        cp_async16(xs + (size_t)r * ld + se_pos<NR>(k), src + (size_t)r * K + k);
    }
    asm volatile("cp.async.commit_group;\n cp.async.wait_all;" ::: "memory");
}

// MODE 0: gate/up + SwiGLU -> h. MODE 1: down -> w * s_d * y per pair.
template <int MODE>
__global__ void __launch_bounds__(kSeThreads, 1) small_expert_kernel(Params p) {
    constexpr int NR = MODE == 0 ? kSeGuRounds : kSeDnRounds;
    extern __shared__ __align__(16) uint8_t se_sm[];
    __shared__ int s_item;
    const int nse = p.cnt[kCntSmall];
    const int H = p.H, I = p.I;
    const int Kin = MODE == 0 ? H : I;              // length of a staged row
    const int C = se_chunks(Kin, NR);               // chunks per weight row
    const int units = MODE == 0 ? I / 8 : H / 16;   // granules per expert
    const int kb = Kin / 2, ks = Kin / 16;          // code, scale bytes per weight row
    const int ld = se_ld(Kin, NR);
    __half *xs = reinterpret_cast<__half *>(se_sm);
    float *fs = reinterpret_cast<float *>(se_sm + (size_t)(kSmallTok + 1) * ld * 2);   // [2][kSmallTok]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const uint8_t *sbase_a = MODE == 0 ? p.gate_scales : p.down_scales;
    const uint8_t *sbase_b = MODE == 0 ? p.up_scales : p.down_scales;
    const bool vec = ks % (2 * NR) == 0 && ((uintptr_t)sbase_a | (uintptr_t)sbase_b) % (2 * NR) == 0;
    const uint8_t *cbase_a = MODE == 0 ? p.gate_codes : p.down_codes;
    const uint8_t *cbase_b = MODE == 0 ? p.up_codes : p.down_codes;
    const bool v32 = kb % 32 == 0 && ((uintptr_t)cbase_a | (uintptr_t)cbase_b) % 32 == 0;
    const bool full = v32 && vec && Kin % (128 * NR) == 0;
    const int S = se_pieces(nse, units, gridDim.x);
    if (nse > 0) {
        uint4 *z = reinterpret_cast<uint4 *>(se_sm);
        for (size_t i = threadIdx.x; i < se_smem(Kin, NR) / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    }
    int bad = -1;
    for (;;) {
        // the next item; the barrier also ends every warp's use of the previous
        // item's rows and factors
        if (threadIdx.x == 0) s_item = atomicAdd(p.cnt + kCntSmallQ + MODE, 1);
        __syncthreads();
        const int it = s_item;
        if (it >= nse * S) break;
        const int u = it / S, piece = it - u * S;
        const int e = p.small_e[u], n = p.counts[e], pos0 = p.offsets[e];
        int ia, ib, wa, wb;
        share(units, piece, S, ia, ib);
        share(ib - ia, warp, kSeWarps, wa, wb);
        // this warp's units: (granule, chunk), granules [ia + wa, ia + wb), walked
        // by two cursors (the chunk computed and the chunk issued two ahead)
        int x = (ia + wa) * C;
        const int end = (ia + wb) * C;
        int cgr = ia + wa, cc = 0, igr = ia + wa, ic = 0;
        // chunk `c` of granule `gr`: gate/up: gate and up rows of intermediate
        // 8 gr + g; down: hidden rows 16 gr + g and + 8
        // the expert's planes; row r of granule gr: gate/up: gate and up rows of
        // intermediate 8 gr + g; down: hidden rows 16 gr + g and + 8
        const size_t rows_e = MODE == 0 ? (size_t)e * I : (size_t)e * H;
        const uint8_t *ca_e = (MODE == 0 ? p.gate_codes : p.down_codes) + rows_e * kb;
        const uint8_t *cb_e = (MODE == 0 ? p.up_codes : p.down_codes) + rows_e * kb;
        const uint8_t *sa_e = sbase_a + rows_e * ks, *sb_e = sbase_b + rows_e * ks;
        const int rstep = MODE == 0 ? 8 : 16, roff_b = MODE == 0 ? 0 : 8;
        // issues the chunk at the issue cursor into b and advances the cursor
        auto issue = [&](SeBuf<NR> &b) {
            const int ra = rstep * igr + g, rb = ra + roff_b;
            se_issue<NR>(ic, ca_e + ra * kb, cb_e + rb * kb, sa_e + ra * ks, sb_e + rb * ks, kb, v32, vec, full, q, b);
            if (++ic == C) {
                ic = 0;
                igr++;
            }
        };
        // three chunk buffers: two chunks in flight while one is computed
        SeBuf<NR> b0, b1, b2;
        if (x < end) issue(b0);   // in flight while the rows are staged
        if (x + 1 < end) issue(b1);
        se_stage<NR>(xs, (MODE == 0 ? p.xh + (size_t)pos0 * H : p.h + (size_t)pos0 * I), n, Kin);
        if (threadIdx.x < kSmallTok) {
            // epilogue factors of pair slot t: gate/up: s_g * x's staging factor and
            // s_u * that * 2^hexp; down: routing weight * s_d
            const int t = threadIdx.x;
            float f0 = 0.0f, f1 = 0.0f;
            if (t < n) {
                const int pos = pos0 + t;
                if (MODE == 0) {
                    const float xsf = p.ps[pos];
                    f0 = p.gate_global[e] * xsf;
                    f1 = p.up_global[e] * (xsf * p.ph[pos]);
                } else {
                    f0 = p.pw[pos] * p.down_global[e];
                }
            }
            fs[t] = f0;
            fs[kSmallTok + t] = f1;
        }
        __syncthreads();
        const int q2 = 2 * q;
        const uint32_t x0 = smem_u32(xs + (size_t)(g < n ? g : kSmallTok) * ld + 32 * NR * q);
        const uint32_t x1 = smem_u32(xs + (size_t)(8 + g < n ? 8 + g : kSmallTok) * ld + 32 * NR * q);
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        // granule done: its outputs for the pairs present (this thread: slots 2q + c
        // of half 0 and 8 + 2q + c of half 1)
        auto finish = [&](int gr) {
            const float a[2][4] = {{acc0[0], acc0[1], acc0[2], acc0[3]}, {acc1[0], acc1[1], acc1[2], acc1[3]}};
#pragma unroll
            for (int hh = 0; hh < 2; hh++)
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const int slot = 8 * hh + 2 * q + c;
                    if (slot < n) {
                        const size_t pos = (size_t)pos0 + slot;
                        if (MODE == 0) {
                            // row g: gate, row g+8: up, of intermediate 8 gr + g
                            const float hf = silu(a[hh][c] * fs[slot]) * (a[hh][2 + c] * fs[kSmallTok + slot]);
                            if (!fits_f16(hf)) bad = e;
                            p.h[pos * I + 8 * gr + g] = __float2half_rn(hf);
                        } else {
                            const float cf = fs[slot];
                            const float y0 = a[hh][c] * cf, y1 = a[hh][2 + c] * cf;
                            if (!fits_f16(y0) || !fits_f16(y1)) bad = e;
                            p.xh[pos * H + 16 * gr + g] = __float2half_rn(y0);
                            p.xh[pos * H + 16 * gr + g + 8] = __float2half_rn(y1);
                        }
                    }
                }
#pragma unroll
            for (int c = 0; c < 4; c++) acc0[c] = acc1[c] = 0.0f;
        };
        // computes chunk x from b; issues chunk x + 2 into nb (computed a step ago)
        auto step = [&](SeBuf<NR> &b, SeBuf<NR> &nb) {
            if (x + 2 < end) issue(nb);
            const uint32_t y0 = x0 + 256 * NR * cc, y1 = x1 + 256 * NR * cc;
#pragma unroll
            for (int j = 0; j < NR; j++)
                se_round(acc0, acc1, b.ca[j], b.cb[j], b.sa[j / 2] >> (16 * (j & 1)), b.sb[j / 2] >> (16 * (j & 1)),
                         y0, y1, j, q2);
            if (++cc == C) {
                finish(cgr);
                cc = 0;
                cgr++;
            }
            x++;
        };
        while (x < end) {
            step(b0, b2);
            if (x >= end) break;
            step(b1, b0);
            if (x >= end) break;
            step(b2, b1);
        }
    }
    warp_report(p, bad, MODE == 0 ? kNfH : kNfY);
    // complete only after the tile kernel this grid was launched behind, so that
    // the launches after it on the stream see both grids' outputs
    grid_dep_wait();
}

int sm_count();   // SMs of the current device (decode.cu)

// Shared memory a small-expert kernel may take (the dynamic part; the kernel
// also has a few bytes of static shared memory).
constexpr int kSeSmemMax = 200 * 1024;

cudaError_t small_init() {
    cudaError_t e = cudaFuncSetAttribute(small_expert_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSeSmemMax);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(small_expert_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSeSmemMax);
    return e;
}

// Whether the small-expert path fits shared memory for these dimensions.
bool small_fits(int H, int I) {
    return se_smem(H, kSeGuRounds) <= kSeSmemMax && se_smem(I, kSeDnRounds) <= kSeSmemMax;
}

cudaError_t launch_small(int mode, const Params &p, cudaStream_t s) {
    if (p.small_tok <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sm_count());
    cfg.blockDim = dim3(kSeThreads);
    cfg.dynamicSmemBytes = mode == 0 ? se_smem(p.H, kSeGuRounds) : se_smem(p.I, kSeDnRounds);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return mode == 0 ? cudaLaunchKernelEx(&cfg, small_expert_kernel<0>, p)
                     : cudaLaunchKernelEx(&cfg, small_expert_kernel<1>, p);
}

}  // namespace nvmoe
