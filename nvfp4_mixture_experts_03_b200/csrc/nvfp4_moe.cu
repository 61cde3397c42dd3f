// Host side of the C ABI declared in include/nvfp4_moe.h: argument validation
// (all of it before any allocation or launch), the workspace layout, TMA tensor
// maps for the grouped GEMMs, and the launch sequence of one forward call.
//
// Conventions follow the pages' readers ("#1858 ... strata-safetensors",
// "Proposed contribution": bounded caller-owned buffers; "TensorFold PR #906",
// first post: complete validation before allocation, nothing left allocated on
// failure): the caller owns every buffer, including the workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "common.cuh"

using namespace nvmoe;

struct nvfp4_moe {
    nvfp4_moe_dims d;
    nvfp4_moe_weights w;
    int device;
    int num_sms;
    int pf_clusters;  // resident CTA pairs of the prefill GEMMs
    CodeMaps codes;   // tensor maps of the weight code planes (prefill GEMMs)
    int32_t *status;  // kStatusWords ints on the device
    uint8_t *dstate;  // decode state (counters, zero between launches), or null
    size_t dstate_bytes;
    int32_t test_flags;  // NVFP4_MOE_TEST_* (test hooks)
    int32_t last_detail; // detail word of the status the last get_status returned
    cudaEvent_t phase[NVFP4_MOE_PHASE_EVENTS];
    bool phase_on;
};

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D F16 tensor [rows][cols], box 64 columns x box_rows, 128-byte swizzle, zero
// fill outside.
bool make_map_f16(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// F16 [rows][cols] as a bulk-store target: unswizzled boxes of box_cols x
// box_rows, laid out in shared memory row after row.
bool make_map_f16_store(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_cols,
                        int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed E2M1 code plane [rows][cols] bytes: 128-byte x box_rows boxes, swizzled
// like the GEMM's shared-memory tiles.
bool make_map_codes(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// Test hook: the n-th device allocation of later creates fails (then disarms).
int g_fail_alloc = 0;
cudaError_t dev_alloc(void **p, size_t bytes) {
    if (g_fail_alloc > 0 && --g_fail_alloc == 0) {
        *p = nullptr;
        return cudaErrorMemoryAllocation;
    }
    return cudaMalloc(p, bytes);
}
inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

// Whether a call with T tokens takes the decode kernel (else the grouped GEMMs).
bool use_decode(const nvfp4_moe_dims &d, int T) {
    return T <= NVFP4_MOE_DECODE_MAX_T && decode_fits(d.hidden, d.inter, d.top_k, d.n_experts);
}

struct WsLayout {
    size_t cnt, ids, wts, hist, cbase, counts, offsets, perm, inv, ptok, pw, ps, xscale, ph, phinv, tiles_gu,
        tiles_dn, small_e, xh, h, rlogits, total;
    int nch, max_gu, max_dn;
};

WsLayout layout(const nvfp4_moe_dims &d, int T) {
    WsLayout L{};
    const size_t P = (size_t)T * d.top_k;
    const int E = d.n_experts;
    L.nch = cdiv(T > 0 ? T : 1, kChunkTokens);
    const bool decode = use_decode(d, T);
    const size_t ntile_n = P / kBN + (size_t)(E < (int)P ? E : (int)P) + 1;
    L.max_gu = decode ? 0 : (int)(ntile_n * cdiv(d.inter, kGuRows));
    L.max_dn = decode ? 0 : (int)(ntile_n * cdiv(d.hidden, kDnRows));
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = a256(o + bytes);
        return at;
    };
    L.cnt = take(kCntWords * 4);
    L.ids = take(P * 4);
    L.wts = take(P * 4);
    L.hist = take(decode ? 0 : (size_t)E * L.nch * 4);
    L.cbase = take(decode ? 0 : (size_t)E * L.nch * 4);
    L.counts = take((size_t)E * 4);
    L.offsets = take((size_t)(E + 1) * 4);
    L.perm = take(P * 4);
    L.inv = take(P * 4);
    L.ptok = take(P * 4);
    L.pw = take(P * 4);
    L.ps = take(P * 4);
    L.xscale = take((size_t)T * 4);
    L.ph = take(decode ? 0 : P * 4);
    L.phinv = take(decode ? 0 : (size_t)T * 4);
    L.tiles_gu = take((size_t)L.max_gu * sizeof(Tile));
    L.tiles_dn = take((size_t)L.max_dn * sizeof(Tile));
    L.small_e = take(decode ? 0 : (size_t)E * 4);
    L.xh = take(decode ? 0 : P * d.hidden * 2);   // decode stages activations in shared memory
    L.h = take(P * d.inter * 2);
    L.rlogits = take((size_t)T * E * 4);   // router projection output (when used)
    L.total = o;
    return L;
}

}  // namespace

extern "C" {

int nvfp4_moe_abi_version(void) { return NVFP4_MOE_ABI_VERSION; }

const char *nvfp4_moe_strerror(int s) {
    switch (s) {
        case NVFP4_MOE_OK: return "ok";
        case NVFP4_MOE_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_MOE_ERR_UNSUPPORTED_DIMS: return "unsupported dimensions";
        case NVFP4_MOE_ERR_MISALIGNED: return "misaligned pointer";
        case NVFP4_MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case NVFP4_MOE_ERR_CUDA: return "CUDA error";
        case NVFP4_MOE_ERR_BAD_ROUTING: return "routing id out of range or repeated";
        case NVFP4_MOE_ERR_NONFINITE: return "non-finite routing logit or computed value";
        case NVFP4_MOE_ERR_TIMEOUT: return "device wait timed out";
        case NVFP4_MOE_ERR_NO_DEVICE: return "no sm_100 device";
        default: return "unknown status";
    }
}

int nvfp4_moe_create(nvfp4_moe_t **out, const nvfp4_moe_dims *dims,
                     const nvfp4_moe_weights *w) {
    if (!out) return NVFP4_MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!dims || !w) return NVFP4_MOE_ERR_INVALID_ARG;
    const nvfp4_moe_dims d = *dims;
    if (d.hidden <= 0 || d.inter <= 0 || d.n_experts <= 0 || d.top_k <= 0 || d.max_tokens < 0)
        return NVFP4_MOE_ERR_INVALID_ARG;
    if (d.hidden % 32 || d.inter % 32 || d.top_k > d.n_experts ||
        d.top_k > NVFP4_MOE_MAX_TOPK || d.n_experts > 1024)
        return NVFP4_MOE_ERR_UNSUPPORTED_DIMS;
    if (d.max_tokens > NVFP4_MOE_MAX_TOKENS) return NVFP4_MOE_ERR_UNSUPPORTED_DIMS;
    const void *planes[] = {w->gate_codes, w->up_codes, w->gate_scales, w->up_scales,
                            w->down_codes, w->down_scales};
    const void *globals[] = {w->gate_global, w->up_global, w->down_global};
    for (const void *p : planes)
        if (!p) return NVFP4_MOE_ERR_INVALID_ARG;
    for (const void *p : globals)
        if (!p) return NVFP4_MOE_ERR_INVALID_ARG;
    for (const void *p : planes)
        if (!al16(p)) return NVFP4_MOE_ERR_MISALIGNED;
    for (const void *p : globals)
        if (!al4(p)) return NVFP4_MOE_ERR_MISALIGNED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_MOE_ERR_NO_DEVICE;
    int major = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10) return NVFP4_MOE_ERR_NO_DEVICE;
    int pf_clusters = 0;
    if (prefill_init(&pf_clusters) != cudaSuccess || decode_init() != cudaSuccess ||
        router_init() != cudaSuccess || small_init() != cudaSuccess || !encode_fn())
        return NVFP4_MOE_ERR_CUDA;
    nvfp4_moe *h = new (std::nothrow) nvfp4_moe;
    if (!h) return NVFP4_MOE_ERR_CUDA;
    h->d = d;
    h->w = *w;
    h->device = dev;
    h->num_sms = sms;
    h->pf_clusters = pf_clusters;
    const int64_t E = d.n_experts;
    if (!make_map_codes(&h->codes.gate, w->gate_codes, E * d.inter, d.hidden / 2, 64) ||
        !make_map_codes(&h->codes.up, w->up_codes, E * d.inter, d.hidden / 2, 64) ||
        !make_map_codes(&h->codes.down, w->down_codes, E * d.hidden, d.inter / 2, 128)) {
        delete h;
        return NVFP4_MOE_ERR_CUDA;
    }
    h->status = nullptr;
    h->dstate = nullptr;
    h->phase_on = false;
    h->test_flags = 0;
    h->last_detail = 0;
    h->dstate_bytes = d.max_tokens >= 1 && use_decode(d, 1) ? decode_state_bytes() : 0;
    if (dev_alloc(reinterpret_cast<void **>(&h->status), kStatusWords * sizeof(int32_t)) != cudaSuccess ||
        cudaMemset(h->status, 0, kStatusWords * sizeof(int32_t)) != cudaSuccess ||
        (h->dstate_bytes &&
         (dev_alloc(reinterpret_cast<void **>(&h->dstate), h->dstate_bytes) != cudaSuccess ||
          cudaMemset(h->dstate, 0, h->dstate_bytes) != cudaSuccess))) {
        if (h->status) cudaFree(h->status);
        if (h->dstate) cudaFree(h->dstate);
        delete h;
        return NVFP4_MOE_ERR_CUDA;
    }
    *out = h;
    return NVFP4_MOE_OK;
}

size_t nvfp4_moe_workspace_bytes(const nvfp4_moe_t *h, int32_t T) {
    if (!h || T < 0 || T > h->d.max_tokens) return 0;
    return layout(h->d, T).total;
}

// Checks a forward call and fills its kernel parameters (everything but the
// launches). Returns NVFP4_MOE_OK, kNothingToDo for T = 0, or an error.
constexpr int kNothingToDo = 1;
static int prepare_forward(nvfp4_moe_t *h, const nvfp4_moe_io *io, void *ws, size_t ws_bytes, Params &p,
                           bool &decode, bool &router) {
    if (!h || !io) return NVFP4_MOE_ERR_INVALID_ARG;
    const nvfp4_moe_dims &d = h->d;
    const int T = io->T;
    if (T < 0 || T > d.max_tokens) return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->act_type != NVFP4_MOE_ACT_BF16 && io->act_type != NVFP4_MOE_ACT_INT8 &&
        io->act_type != NVFP4_MOE_ACT_F32)
        return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->out_type != NVFP4_MOE_OUT_F32 && io->out_type != NVFP4_MOE_OUT_F32_ADD)
        return NVFP4_MOE_ERR_INVALID_ARG;
    if (T == 0) return kNothingToDo;
    if (!io->act || !io->out) return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->act_type == NVFP4_MOE_ACT_INT8 && !io->act_scale) return NVFP4_MOE_ERR_INVALID_ARG;
    // routing source: given logits, the router projection, or given ids and weights
    router = !io->router_logits && io->router_w;
    if (io->router_logits && io->router_w) return NVFP4_MOE_ERR_INVALID_ARG;
    if (router && (io->topk_ids || io->topk_weights)) return NVFP4_MOE_ERR_INVALID_ARG;
    if (!io->router_logits && !router && (!io->topk_ids || !io->topk_weights)) return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->act == io->out && io->out_type != NVFP4_MOE_OUT_F32_ADD) return NVFP4_MOE_ERR_INVALID_ARG;
    if (!al16(io->act) || !al16(io->out) || (io->router_logits && !al16(io->router_logits)) ||
        (io->act_scale && !al4(io->act_scale)) || (io->topk_ids && !al4(io->topk_ids)) ||
        (io->topk_weights && !al4(io->topk_weights)) || (io->router_w && !al16(io->router_w)) ||
        (io->dbg_logits && !al16(io->dbg_logits)))
        return NVFP4_MOE_ERR_MISALIGNED;
    const WsLayout L = layout(d, T);
    if (!ws || ws_bytes < L.total) return NVFP4_MOE_ERR_WORKSPACE_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return NVFP4_MOE_ERR_MISALIGNED;

    uint8_t *b = static_cast<uint8_t *>(ws);
    p = Params{};
    p.T = T;
    p.E = d.n_experts;
    p.H = d.hidden;
    p.I = d.inter;
    p.K = d.top_k;
    p.act_type = io->act_type;
    p.out_add = io->out_type == NVFP4_MOE_OUT_F32_ADD;
    p.act = io->act;
    p.act_scale = io->act_scale;
    p.logits = io->router_logits;
    p.router_w = io->router_w;
    p.rlogits = io->dbg_logits ? io->dbg_logits : reinterpret_cast<float *>(b + L.rlogits);
    if (router) p.logits = p.rlogits;
    p.in_ids = io->topk_ids;
    p.in_w = io->topk_weights;
    p.out = io->out;
    p.gate_codes = h->w.gate_codes;
    p.up_codes = h->w.up_codes;
    p.gate_scales = h->w.gate_scales;
    p.up_scales = h->w.up_scales;
    p.gate_global = h->w.gate_global;
    p.up_global = h->w.up_global;
    p.down_codes = h->w.down_codes;
    p.down_scales = h->w.down_scales;
    p.down_global = h->w.down_global;
    p.cnt = reinterpret_cast<int32_t *>(b + L.cnt);
    p.ids = reinterpret_cast<int32_t *>(b + L.ids);
    p.wts = reinterpret_cast<float *>(b + L.wts);
    p.hist = reinterpret_cast<int32_t *>(b + L.hist);
    p.cbase = reinterpret_cast<int32_t *>(b + L.cbase);
    p.counts = reinterpret_cast<int32_t *>(b + L.counts);
    p.offsets = reinterpret_cast<int32_t *>(b + L.offsets);
    p.perm = reinterpret_cast<int32_t *>(b + L.perm);
    p.inv = reinterpret_cast<int32_t *>(b + L.inv);
    p.ptok = reinterpret_cast<int32_t *>(b + L.ptok);
    p.pw = reinterpret_cast<float *>(b + L.pw);
    p.ps = reinterpret_cast<float *>(b + L.ps);
    p.xscale = reinterpret_cast<float *>(b + L.xscale);
    p.ph = reinterpret_cast<float *>(b + L.ph);
    p.phinv = reinterpret_cast<float *>(b + L.phinv);
    p.tiles_gu = reinterpret_cast<Tile *>(b + L.tiles_gu);
    p.tiles_dn = reinterpret_cast<Tile *>(b + L.tiles_dn);
    p.small_e = reinterpret_cast<int32_t *>(b + L.small_e);
    p.small_tok = (h->test_flags & NVFP4_MOE_TEST_NO_SMALL) || !small_fits(d.hidden, d.inter) ? 0 : kSmallTok;
    p.xh = reinterpret_cast<__half *>(b + L.xh);
    p.h = reinterpret_cast<__half *>(b + L.h);
    p.status = h->status;
    p.dbg_ids = io->dbg_ids;
    p.dbg_w = io->dbg_w;
    p.dbg_counts = io->dbg_counts;
    p.dbg_offsets = io->dbg_offsets;
    p.dbg_perm = io->dbg_perm;
    p.nch = L.nch;
    p.max_tiles_gu = L.max_gu;
    p.max_tiles_dn = L.max_dn;
    p.test_flags = h->test_flags;
    decode = use_decode(d, T);
    if (decode) {
        if (!h->dstate) return NVFP4_MOE_ERR_INVALID_ARG;
        p.dstate = reinterpret_cast<int32_t *>(h->dstate);
        p.dec_union = (int32_t)decode_union_bytes(T, d.top_k, d.hidden, d.inter);
    }

    return NVFP4_MOE_OK;
}

int nvfp4_moe_forward(nvfp4_moe_t *h, const nvfp4_moe_io *io, void *ws, size_t ws_bytes,
                      void *stream) {
    Params p;
    bool decode = false, router = false;
    const int pr = prepare_forward(h, io, ws, ws_bytes, p, decode, router);
    if (pr == kNothingToDo) return NVFP4_MOE_OK;
    if (pr != NVFP4_MOE_OK) return pr;
    const nvfp4_moe_dims &d = h->d;
    const int T = io->T;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // External records, so that a forward captured into a CUDA graph records the
    // phase events on every replay (a plain record inside capture is only an
    // ordering dependency).
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (h->phase_on && cudaStreamIsCapturing(s, &cap) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
    auto mark = [&](int i) {
        if (!h->phase_on) return;
        if (cap == cudaStreamCaptureStatusActive)
            cudaEventRecordWithFlags(h->phase[i], s, cudaEventRecordExternal);
        else
            cudaEventRecord(h->phase[i], s);
    };
    if (decode) {
        // one kernel for the whole decode layer: its routing, staging and both
        // projections are not separable by events (phases 0-2 and 3-4 coincide)
        mark(0);
        if (router && launch_router(p, s) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
        mark(1);
        mark(2);
        if (launch_decode(p, s) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
        mark(3);
        mark(4);
    } else {
        const int64_t P = (int64_t)T * d.top_k;
        CUtensorMap map_xh, map_h, map_y;
        if (!make_map_f16(&map_xh, p.xh, P, d.hidden, 64) || !make_map_f16(&map_h, p.h, P, d.inter, 64) ||
            !make_map_f16_store(&map_y, p.xh, P, d.hidden, 128, 32))
            return NVFP4_MOE_ERR_CUDA;
        mark(0);
        if (router && launch_router(p, s) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
        launch_route_large(p, s);
        mark(1);
        launch_prep_prefill(p, s);
        mark(2);
        if (launch_prefill_gemm(0, p, map_xh, h->codes, map_y, h->pf_clusters, s) != cudaSuccess ||
            launch_small(0, p, s) != cudaSuccess)
            return NVFP4_MOE_ERR_CUDA;
        mark(3);
        if (launch_prefill_gemm(1, p, map_h, h->codes, map_y, h->pf_clusters, s) != cudaSuccess ||
            launch_small(1, p, s) != cudaSuccess)
            return NVFP4_MOE_ERR_CUDA;
        launch_combine(p, s);
        mark(4);
    }
    return cudaGetLastError() == cudaSuccess ? NVFP4_MOE_OK : NVFP4_MOE_ERR_CUDA;
}

int nvfp4_moe_forward_decode_stack(nvfp4_moe_t *const *layers, int32_t n_layers, const nvfp4_moe_io *io,
                                   void *ws, size_t ws_bytes, void *stream) {
    if (!layers || !io || n_layers < 1 || n_layers > NVFP4_MOE_MAX_STACK) return NVFP4_MOE_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; l++) {
        if (!layers[l]) return NVFP4_MOE_ERR_INVALID_ARG;
        const nvfp4_moe_dims &a = layers[l]->d, &b0 = layers[0]->d;
        if (a.hidden != b0.hidden || a.inter != b0.inter || a.n_experts != b0.n_experts ||
            a.top_k != b0.top_k || layers[l]->device != layers[0]->device)
            return NVFP4_MOE_ERR_INVALID_ARG;
        if (io->T > a.max_tokens) return NVFP4_MOE_ERR_INVALID_ARG;
    }
    // the residual stream in place, routed from per-layer logits
    if (io->act_type != NVFP4_MOE_ACT_F32 || io->out_type != NVFP4_MOE_OUT_F32_ADD || io->act != io->out ||
        !io->router_logits || io->router_w || io->topk_ids || io->topk_weights)
        return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->dbg_ids || io->dbg_w || io->dbg_counts || io->dbg_offsets || io->dbg_perm || io->dbg_logits)
        return NVFP4_MOE_ERR_INVALID_ARG;
    Params p;
    bool decode = false, router = false;
    const int pr = prepare_forward(layers[0], io, ws, ws_bytes, p, decode, router);
    if (pr == kNothingToDo) return NVFP4_MOE_OK;
    if (pr != NVFP4_MOE_OK) return pr;
    if (!decode) return NVFP4_MOE_ERR_UNSUPPORTED_DIMS;
    DecLayerPtrs w[NVFP4_MOE_MAX_STACK];
    for (int l = 0; l < n_layers; l++) {
        const nvfp4_moe_weights &x = layers[l]->w;
        w[l] = DecLayerPtrs{x.gate_codes, x.up_codes, x.gate_scales, x.up_scales, x.gate_global,
                            x.up_global, x.down_codes, x.down_scales, x.down_global};
    }
    if (launch_decode_stack(p, w, n_layers, io->router_logits, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return NVFP4_MOE_ERR_CUDA;
    return NVFP4_MOE_OK;
}

int nvfp4_moe_get_status(nvfp4_moe_t *h, void *stream) {
    if (!h) return NVFP4_MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t st[kStatusWords];
    if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
    if (cudaMemcpy(st, h->status, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess)
        return NVFP4_MOE_ERR_CUDA;
    if (cudaMemset(h->status, 0, sizeof(st)) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
    h->last_detail = st[kStatusCode] != 0 ? st[kStatusDetail] : 0;
    // A launch that gave up may have left decode counts behind.
    if (st[kStatusCode] != 0 && h->dstate && cudaMemset(h->dstate, 0, h->dstate_bytes) != cudaSuccess)
        return NVFP4_MOE_ERR_CUDA;
    return st[kStatusCode];
}

int nvfp4_moe_set_phase_events(nvfp4_moe_t *h, void *const *events, int32_t n_events) {
    if (!h) return NVFP4_MOE_ERR_INVALID_ARG;
    if (n_events == 0) {
        h->phase_on = false;
        return NVFP4_MOE_OK;
    }
    if (n_events != NVFP4_MOE_PHASE_EVENTS || !events) return NVFP4_MOE_ERR_INVALID_ARG;
    for (int i = 0; i < NVFP4_MOE_PHASE_EVENTS; i++)
        if (!events[i]) return NVFP4_MOE_ERR_INVALID_ARG;
    for (int i = 0; i < NVFP4_MOE_PHASE_EVENTS; i++) h->phase[i] = static_cast<cudaEvent_t>(events[i]);
    h->phase_on = true;
    return NVFP4_MOE_OK;
}

int nvfp4_moe_test_set_flags(nvfp4_moe_t *h, int32_t flags) {
    if (!h || (flags & ~(NVFP4_MOE_TEST_DECODE_STALL | NVFP4_MOE_TEST_NO_SMALL))) return NVFP4_MOE_ERR_INVALID_ARG;
    h->test_flags = flags;
    return NVFP4_MOE_OK;
}

int nvfp4_moe_test_last_detail(const nvfp4_moe_t *h) { return h ? h->last_detail : 0; }

void nvfp4_moe_test_fail_alloc(int32_t n) { g_fail_alloc = n > 0 ? n : 0; }

void nvfp4_moe_destroy(nvfp4_moe_t *h) {
    if (!h) return;
    if (h->status) cudaFree(h->status);
    if (h->dstate) cudaFree(h->dstate);
    delete h;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode entry point.
//
// For callers that cannot allocate device memory at all -- code running where
// cudaMalloc is forbidden or unavailable (an allocator-less embedding, a process
// whose device memory is fully pre-reserved by another runtime) -- and so can
// neither create a handle (create allocates its status block) nor provide a
// workspace. The decode path's scratch (routing arrays, F16 activations, h)
// lives instead in this file-scope device array, which every GPU that loads the
// library holds until the process exits.
namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB per device
constexpr size_t kStaticStatusBytes = 256;               // status words, then decode state, workspace
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
uint8_t *g_static_ptr[kMaxDevices];  // device address of g_static_scratch, per device

// Per-device set-up, once, with that device current: the array's name is only a
// host-side stand-in, so its device address is looked up here; and the decode
// kernels are opted into the dynamic shared memory they need (above the 48 KB
// default at realistic layer sizes), which a process that never created a handle
// on this device has not done yet. Neither step allocates device memory.
int static_scratch(int dev, uint8_t **out) {
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_MOE_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p)
            return NVFP4_MOE_ERR_CUDA;
        if (decode_init() != cudaSuccess || router_init() != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
        g_static_ptr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_static_ptr[dev];
    return NVFP4_MOE_OK;
}

// The same dims/weights checks as nvfp4_moe_create, without its allocation.
int check_layer(const nvfp4_moe_dims *dims, const nvfp4_moe_weights *w) {
    if (!dims || !w) return NVFP4_MOE_ERR_INVALID_ARG;
    const nvfp4_moe_dims d = *dims;
    if (d.hidden <= 0 || d.inter <= 0 || d.n_experts <= 0 || d.top_k <= 0 || d.max_tokens < 0)
        return NVFP4_MOE_ERR_INVALID_ARG;
    if (d.hidden % 32 || d.inter % 32 || d.top_k > d.n_experts ||
        d.top_k > NVFP4_MOE_MAX_TOPK || d.n_experts > 1024 || d.max_tokens > NVFP4_MOE_MAX_TOKENS)
        return NVFP4_MOE_ERR_UNSUPPORTED_DIMS;
    const void *planes[] = {w->gate_codes, w->up_codes, w->gate_scales, w->up_scales,
                            w->down_codes, w->down_scales};
    const void *globals[] = {w->gate_global, w->up_global, w->down_global};
    for (const void *p : planes)
        if (!p) return NVFP4_MOE_ERR_INVALID_ARG;
    for (const void *p : globals)
        if (!p) return NVFP4_MOE_ERR_INVALID_ARG;
    for (const void *p : planes)
        if (!al16(p)) return NVFP4_MOE_ERR_MISALIGNED;
    for (const void *p : globals)
        if (!al4(p)) return NVFP4_MOE_ERR_MISALIGNED;
    return NVFP4_MOE_OK;
}

}  // namespace

extern "C" {

int nvfp4_moe_forward_decode_static(const nvfp4_moe_dims *dims, const nvfp4_moe_weights *w,
                                    const nvfp4_moe_io *io, void *stream) {
    int rc = check_layer(dims, w);
    if (rc != NVFP4_MOE_OK) return rc;
    if (!io) return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->T < 0 || io->T > dims->max_tokens) return NVFP4_MOE_ERR_INVALID_ARG;
    if (io->T > NVFP4_MOE_DECODE_MAX_T || !use_decode(*dims, io->T)) return NVFP4_MOE_ERR_UNSUPPORTED_DIMS;
    if (io->T == 0) return NVFP4_MOE_OK;
    const size_t state = decode_state_bytes();
    const size_t need = layout(*dims, io->T).total;
    if (need + state > kStaticScratchBytes - kStaticStatusBytes) return NVFP4_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_MOE_ERR_NO_DEVICE;
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        major != 10)
        return NVFP4_MOE_ERR_NO_DEVICE;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint8_t *scratch = nullptr;
    rc = static_scratch(dev, &scratch);
    if (rc != NVFP4_MOE_OK) return rc;
    // A handle on the stack (allocates nothing) pointing at the static array.
    nvfp4_moe h;
    h.d = *dims;
    h.w = *w;
    h.device = dev;
    h.num_sms = sms;
    h.pf_clusters = 0;   // the decode kernel never reaches the prefill GEMMs
    h.test_flags = 0;
    h.last_detail = 0;
    h.status = reinterpret_cast<int32_t *>(scratch);
    h.dstate = scratch + kStaticStatusBytes;
    h.dstate_bytes = state;
    h.phase_on = false;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The status words and the decode counters must start at zero (the status
    // latches the first device error; an earlier call that gave up may have left
    // counts behind, and no status read follows a call here).
    if (cudaMemsetAsync(scratch, 0, kStaticStatusBytes + state, s) != cudaSuccess) return NVFP4_MOE_ERR_CUDA;
    return nvfp4_moe_forward(&h, io, scratch + kStaticStatusBytes + state,
                             kStaticScratchBytes - kStaticStatusBytes - state, stream);
}

}  // extern "C"
