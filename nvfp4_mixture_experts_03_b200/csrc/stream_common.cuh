// Helpers of the kernels that stream NVFP4 weights through registers into
// mma.sync (the decode layer and the small-expert path of the grouped GEMMs).
#pragma once
#include "common.cuh"

namespace nvmoe {

// 16 bytes that are read once: no L1 allocation.
__device__ inline uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 32 bytes that are read once (a 32-byte aligned address): no L1 allocation.
__device__ inline void ldg_stream32(const void *p, uint4 &lo, uint4 &hi) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
}

// 16-byte asynchronous copy global -> shared (L2 only).
__device__ inline void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}

// [a, b) = worker w's share of n units when W workers split them evenly in
// contiguous ranges.
__device__ inline void share(int n, int w, int W, int &a, int &b) {
    a = (int)((long long)n * w / W);
    b = (int)((long long)n * (w + 1) / W);
}

// Latches NONFINITE (detail: stage | expert or row) if any lane of the warp saw
// a bad value.
__device__ inline void warp_report(const Params &p, int bad, int stage) {
    const unsigned m = __ballot_sync(0xffffffffu, bad >= 0);
    if (m) {
        const int v = __shfl_sync(0xffffffffu, bad, __ffs(m) - 1);
        if ((threadIdx.x & 31) == 0) latch_status(p.status, NVFP4_MOE_ERR_NONFINITE, stage | v);
    }
}

}  // namespace nvmoe
