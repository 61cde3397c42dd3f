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
constexpr int kRoundsInFlight = 4;

// gate/up + SwiGLU. Item = (unique expert u, 8 intermediate rows): A rows g are
// gate rows, rows g+8 the up rows of the same intermediate index, so each
// thread ends with g and u of the same (row, token) pair.
__global__ void __launch_bounds__(kDecWarps * 32, 2) decode_gateup_kernel(Params p) {
    extern __shared__ __align__(16) __half xs[];  // [8][H+4]
    const int H = p.H, I = p.I, ld = H + 4;
    const int T = p.T;
    for (int idx = threadIdx.x; idx < 8 * (H / 4); idx += blockDim.x) {
        const int tok = idx / (H / 4), k4 = idx % (H / 4);
        uint2 v = make_uint2(0, 0);
        if (tok < T) v = reinterpret_cast<const uint2 *>(p.xh + (size_t)tok * H)[k4];
        *reinterpret_cast<uint2 *>(xs + tok * ld + 4 * k4) = v;
    }
    __syncthreads();
    const int U = p.cnt[kCntUniq];
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int items = U * (I / 8);
    const int rounds = H / 128;
    const __half *xrow = xs + g * ld + 32 * q;
    for (int item = blockIdx.x * kDecWarps + (threadIdx.x >> 5); item < items;
         item += gridDim.x * kDecWarps) {
        const int u = item / (I / 8), i0 = (item % (I / 8)) * 8;
        const int e = p.uniq[u];
        const size_t ra = (size_t)e * I + i0 + g;
        const uint8_t *ga = p.gate_codes + ra * (H / 2) + 16 * q;
        const uint8_t *ua = p.up_codes + ra * (H / 2) + 16 * q;
        const uint8_t *gs = p.gate_scales + ra * (H / 16) + 2 * q;
        const uint8_t *us = p.up_scales + ra * (H / 16) + 2 * q;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int r0 = 0; r0 < rounds; r0 += kRoundsInFlight) {
            uint4 cg[kRoundsInFlight], cu[kRoundsInFlight];
            uint32_t sg[kRoundsInFlight], su[kRoundsInFlight];
#pragma unroll
            for (int j = 0; j < kRoundsInFlight; j++) {
                if (r0 + j < rounds) {
                    const int r = r0 + j;
                    cg[j] = ldg_stream(ga + 64 * r);
                    cu[j] = ldg_stream(ua + 64 * r);
                    sg[j] = __ldg(reinterpret_cast<const unsigned short *>(gs + 8 * r));
                    su[j] = __ldg(reinterpret_cast<const unsigned short *>(us + 8 * r));
                }
            }
#pragma unroll
            for (int j = 0; j < kRoundsInFlight; j++) {
                if (r0 + j < rounds) {
                    const __half *xr = xrow + 128 * (r0 + j);
                    round_mma(acc, cg[j], cu[j], sg[j], su[j],
                              [&](int s, uint32_t &x0, uint32_t &x1) {
                                  const uint2 v = *reinterpret_cast<const uint2 *>(xr + 4 * s);
                                  x0 = v.x;
                                  x1 = v.y;
                              });
                }
            }
        }
        const float sgl = p.gate_global[e], sul = p.up_global[e];
#pragma unroll
        for (int c = 0; c < 2; c++) {
            const int tok = 2 * q + c;
            if (tok < T) {
                const int pos = p.upos[u * NVFP4_MOE_DECODE_MAX_T + tok];
                if (pos >= 0) {
                    const float xsc = p.xscale[tok];
                    const float gv = acc[c] * sgl * xsc, uv = acc[2 + c] * sul * xsc;
                    p.h[(size_t)pos * I + i0 + g] = __float2half_rn(silu(gv) * uv);
                }
            }
        }
    }
}

// down + weighted combine. Item = (unique expert u, 16 hidden rows). B operand:
// h of the pairs (token, u); tokens not routed to u contribute zeros.
__global__ void __launch_bounds__(kDecWarps * 32, 2) decode_down_kernel(Params p) {
    const int H = p.H, I = p.I, T = p.T;
    const int U = p.cnt[kCntUniq];
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int items = U * (H / 16);
    const int rounds = I / 128;
    for (int item = blockIdx.x * kDecWarps + (threadIdx.x >> 5); item < items;
         item += gridDim.x * kDecWarps) {
        const int u = item / (H / 16), m0 = (item % (H / 16)) * 16;
        const int e = p.uniq[u];
        const size_t ra = (size_t)e * H + m0 + g;
        const uint8_t *da = p.down_codes + ra * (I / 2) + 16 * q;
        const uint8_t *db = p.down_codes + (ra + 8) * (I / 2) + 16 * q;
        const uint8_t *sa_p = p.down_scales + ra * (I / 16) + 2 * q;
        const uint8_t *sb_p = p.down_scales + (ra + 8) * (I / 16) + 2 * q;
        const int mypos = (g < T) ? p.upos[u * NVFP4_MOE_DECODE_MAX_T + g] : -1;
        const __half *hrow = p.h + (size_t)(mypos < 0 ? 0 : mypos) * I + 32 * q;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int r0 = 0; r0 < rounds; r0 += kRoundsInFlight) {
            uint4 ca[kRoundsInFlight], cb[kRoundsInFlight];
            uint32_t sa[kRoundsInFlight], sb[kRoundsInFlight];
            uint4 hv[kRoundsInFlight][4];
#pragma unroll
            for (int j = 0; j < kRoundsInFlight; j++) {
                if (r0 + j < rounds) {
                    const int r = r0 + j;
                    ca[j] = ldg_stream(da + 64 * r);
                    cb[j] = ldg_stream(db + 64 * r);
                    sa[j] = __ldg(reinterpret_cast<const unsigned short *>(sa_p + 8 * r));
                    sb[j] = __ldg(reinterpret_cast<const unsigned short *>(sb_p + 8 * r));
#pragma unroll
                    for (int v = 0; v < 4; v++)
                        hv[j][v] = mypos >= 0
                                       ? reinterpret_cast<const uint4 *>(hrow + 128 * r)[v]
                                       : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int j = 0; j < kRoundsInFlight; j++) {
                if (r0 + j < rounds) {
                    round_mma(acc, ca[j], cb[j], sa[j], sb[j],
                              [&](int s, uint32_t &x0, uint32_t &x1) {
                                  // 4 halves at 4s..4s+3 of this thread's 32
                                  const uint4 &w = hv[j][s >> 1];
                                  x0 = (s & 1) ? w.z : w.x;
                                  x1 = (s & 1) ? w.w : w.y;
                              });
                }
            }
        }
        const float sd = p.down_global[e];
#pragma unroll
        for (int c = 0; c < 2; c++) {
            const int tok = 2 * q + c;
            if (tok < T) {
                const int pos = p.upos[u * NVFP4_MOE_DECODE_MAX_T + tok];
                if (pos >= 0) {
                    const float w = p.pw[pos] * sd;
                    atomicAdd(p.out + (size_t)tok * H + m0 + g, acc[c] * w);
                    atomicAdd(p.out + (size_t)tok * H + m0 + g + 8, acc[2 + c] * w);
                }
            }
        }
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
    const size_t xs_bytes = (size_t)8 * (p.H + 4) * sizeof(__half);
    const int items = U_max * (p.I / 8);
    const int grid = max(1, min(2 * sm_count(), cdiv(items, kDecWarps)));
    decode_gateup_kernel<<<grid, kDecWarps * 32, xs_bytes, s>>>(p);
}

void launch_decode_down(const Params &p, cudaStream_t s) {
    const int U_max = min(p.T * p.K, p.E);
    const int items = U_max * (p.H / 16);
    const int grid = max(1, min(2 * sm_count(), cdiv(items, kDecWarps)));
    decode_down_kernel<<<grid, kDecWarps * 32, 0, s>>>(p);
}

}  // namespace nvmoe
