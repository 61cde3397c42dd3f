// Decode path (T <= 8): stream each selected expert's 4.5-bit weights once.
//
// The pages keep the quality profile on "canonical FP32 expert decode" ("#1858
// ... strata-safetensors", "What do you want to do?" and the paragraph after
// the measurements) and note that a decode round is bound by moving expert
// bytes ("Strata NVFP4" README, "Limits"). On B200 every expert is resident in
// HBM, so decode is a pure HBM stream; the arithmetic must stay below ~3 issued
// instructions per weight to keep up. Each weight is decoded exactly to F16
// (E2M1 -> F16 by the hardware conversion, times its E4M3 group scale: the
// product has at most 6 significant bits and is exact in F16) and fed to
// mma.sync m16n8k16 with the (up to 8) tokens as N, accumulating in FP32. The
// tensor scale and the per-token activation scale are applied to the FP32
// result, never folded into F16 operands.
//
// Work item of one warp: 16 weight rows x all K of one selected expert.
// Fragment mapping (m16n8k16, A row-major, B col-major): thread (g = lane/4,
// q = lane%4) holds rows g and g+8. It loads 16 contiguous code bytes of each
// row per 128-wide K round (byte offset 64*r + 16*q), so a warp reads two full
// 32-byte sectors per row per load. Mma step s of round r uses physical K
// 128r + 32q + 4s + {0,1,2,3} for logical K {2q, 2q+1, 2q+8, 2q+9}: the same
// K permutation is applied to the activations, so the dot products are exact.
#include "common.cuh"

namespace nvmoe {

__device__ inline uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

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
constexpr int kMaxRoundsPerWarp = 4;   // 128-wide K rounds of loads one warp holds per pass

// Number of warps that share one item's K range (1, 2 or 4): each warp takes
// rounds/split consecutive rounds; the partial sums meet in shared memory.
__host__ __device__ inline int k_split(int rounds) {
    if (rounds % 4 == 0 && rounds / 4 <= kMaxRoundsPerWarp) return 4;
    if (rounds % 2 == 0 && rounds / 2 <= kMaxRoundsPerWarp) return 2;
    return rounds <= kMaxRoundsPerWarp ? 1 : 4;
}

// One pass's weight data of one warp: rows g and g+8, up to kMaxRoundsPerWarp rounds.
struct PassBuf {
    uint4 ca[kMaxRoundsPerWarp], cb[kMaxRoundsPerWarp];
    uint32_t sa[kMaxRoundsPerWarp], sb[kMaxRoundsPerWarp];
};

struct ItemRef {
    int item, u, e, m0;
    bool valid;
};

template <int MODE>
__device__ inline ItemRef item_ref(const Params &p, int item, int items) {
    ItemRef r{item, 0, 0, 0, item < items};
    if (r.valid) {
        const int per_u = MODE == 0 ? p.I / 8 : p.H / 16;
        r.u = item / per_u;
        r.m0 = (item % per_u) * (MODE == 0 ? 8 : 16);
        r.e = p.uniq[r.u];
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
template <int MODE>
__global__ void __launch_bounds__(kDecWarps * 32, 2) decode_kernel(Params p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    const int H = p.H, I = p.I, T = p.T;
    const int Kd = MODE == 0 ? H : I;
    const int rounds = Kd / 128;
    const int split = k_split(rounds);
    const int rpw = cdiv(rounds, split);               // rounds per warp
    const int ipc = kDecWarps / split;                 // items per CTA pass
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    float *red = reinterpret_cast<float *>(dsm);       // [kDecWarps][32][4]
    __half *xs = reinterpret_cast<__half *>(dsm + kDecWarps * 32 * 4 * sizeof(float));  // [8][H+4]
    const int ld = H + 4;
    const int U = p.cnt[kCntUniq];
    const int items = U * ((MODE == 0 ? I : H) / (MODE == 0 ? 8 : 16));
    const int item_l = warp / split, part = warp % split;
    const int r_begin = part * rpw, r_end = min(rounds, r_begin + rpw);
    const int stride = gridDim.x * ipc;

    PassBuf buf0, buf1;
    int base = blockIdx.x * ipc;
    ItemRef cur = item_ref<MODE>(p, base + item_l, items);
    issue_loads<MODE>(p, cur, g, q, r_begin, r_end, buf0);
    if (MODE == 0) {
        // the F16 activations of all 8 token slots (zeros past T), staged once per
        // CTA while the first pass's weight loads are in flight
        const int n16 = 8 * (H / 8);
#pragma unroll 4
        for (int idx = threadIdx.x; idx < n16; idx += blockDim.x) {
            const int tok = idx / (H / 8), k8 = idx % (H / 8);
            uint4 v = make_uint4(0, 0, 0, 0);
            if (tok < T) v = reinterpret_cast<const uint4 *>(p.xh + (size_t)tok * H)[k8];
            uint2 *d = reinterpret_cast<uint2 *>(xs + tok * ld + 8 * k8);
            d[0] = make_uint2(v.x, v.y);
            d[1] = make_uint2(v.z, v.w);
        }
        __syncthreads();
    }
    const __half *xrow = xs + g * ld + 32 * q;
    // one pass: compute from b while the next pass's loads fill nb
    auto pass_step = [&](PassBuf &b, PassBuf &nb) {
        const ItemRef nxt = item_ref<MODE>(p, base + stride + item_l, items);
        issue_loads<MODE>(p, nxt, g, q, r_begin, r_end, nb);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (cur.valid) {
            int mypos = -1;
            if (MODE == 1 && g < T) mypos = p.upos[cur.u * NVFP4_MOE_DECODE_MAX_T + g];
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
                    if (tok < T) {
                        const int pos = p.upos[cur.u * NVFP4_MOE_DECODE_MAX_T + tok];
                        if (pos >= 0) {
                            const float xsc = p.xscale[tok];
                            const float gv = acc[c] * sgl * xsc, uv = acc[2 + c] * sul * xsc;
                            p.h[(size_t)pos * I + cur.m0 + g] = __float2half_rn(silu(gv) * uv);
                        }
                    }
                }
            } else {
                const float sd = p.down_global[cur.e];
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const int tok = 2 * q + c;
                    if (tok < T) {
                        const int pos = p.upos[cur.u * NVFP4_MOE_DECODE_MAX_T + tok];
                        if (pos >= 0) {
                            const float w = p.pw[pos] * sd;
                            atomicAdd(p.out + (size_t)tok * H + cur.m0 + g, acc[c] * w);
                            atomicAdd(p.out + (size_t)tok * H + cur.m0 + g + 8, acc[2 + c] * w);
                        }
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

void launch_decode_gateup(const Params &p, cudaStream_t s) {
    const int U_max = min(p.T * p.K, p.E);
    const int split = k_split(p.H / 128);
    const int ipc = kDecWarps / split;
    const size_t smem = kDecWarps * 32 * 4 * sizeof(float) + (size_t)8 * (p.H + 4) * sizeof(__half);
    const int items = U_max * (p.I / 8);
    const int grid = max(1, min(2 * sm_count(), cdiv(items, ipc)));
    decode_kernel<0><<<grid, kDecWarps * 32, smem, s>>>(p);
}

void launch_decode_down(const Params &p, cudaStream_t s) {
    const int U_max = min(p.T * p.K, p.E);
    const int split = k_split(p.I / 128);
    const int ipc = kDecWarps / split;
    const size_t smem = kDecWarps * 32 * 4 * sizeof(float);
    const int items = U_max * (p.H / 16);
    const int grid = max(1, min(2 * sm_count(), cdiv(items, ipc)));
    decode_kernel<1><<<grid, kDecWarps * 32, smem, s>>>(p);
}

}  // namespace nvmoe
