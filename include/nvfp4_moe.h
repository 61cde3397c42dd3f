/*
 * nvfp4_moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts FFN layer
 * over ModelOpt-style NVFP4 expert weights.
 *
 * What the layer computes (per token t, top-k experts e_j, j = 0..K-1):
 *
 *   g   = s_g(e) * (G_e x_t)          gate projection,  G_e [I][H]
 *   u   = s_u(e) * (U_e x_t)          up projection,    U_e [I][H]
 *   h   = SiLU(g) * u,  SiLU(z) = z / (1 + exp(-z))
 *   y   = s_d(e) * (D_e h)            down projection,  D_e [H][I]
 *   out_t = sum_j w_{t,j} * y_{t,e_j}
 *
 * Sources on the pages:
 *   - NVFP4 expert weights: 4-bit codes with a scale per group of 16 inputs and
 *     one FP32 tensor scale ("TensorFold PR #906", first post: input cuts keep
 *     groups of 16, the FP32 tensor scale is unchanged; "Strata NVFP4" README,
 *     "How it differs from upstream Strata": 4.5-bit experts with calibrated
 *     scales, lossless repack).
 *   - The per-expert FP32 scale is applied to each projection's OUTPUT, not folded
 *     into the operands ("Strata NVFP4" README, "How it differs", first bullet);
 *     folding a tiny scale into FP16 activations pushed them into FP16 subnormals
 *     (same README, the "Fixes" bullet). This library applies s_g, s_u, s_d in
 *     FP32 after accumulation.
 *   - Routed experts, gate/up/down tensors stacked per layer: "#2727 tools: add
 *     opt-in FP4-Local CSF checkpoint conversion", "Validation" (144 NVFP4 expert
 *     tensors, 512 experts each; nine projection global scales for three experts).
 *   - One launch per expert group after one wait instead of a wait per expert:
 *     "Strata NVFP4" README, "How it differs", the prompt-reading bullet. Every
 *     forward call here is a fixed sequence of launches with no host read-back.
 *   - The pages never write the routing math out. Routing here is softmax top-k,
 *     renormalised over the K selected experts (the tiny-layer workload's
 *     definition); this equals exp(l_j - l_max) / sum over the K selected.
 *
 * Packed formats (all planes row-major, no padding, no swizzle):
 *   E2M1 code nibble: bit 3 sign, bits 2..1 exponent, bit 0 mantissa (OCP MX);
 *     magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. Element 2c of a row is in the LOW
 *     nibble of byte c, element 2c+1 in the HIGH nibble.
 *   E4M3 scale byte (OCP FP8 E4M3FN): bias 7, no infinities, 0x7F/0xFF NaN.
 *     Scales must be finite and non-negative; the layer does not re-check them.
 *   Weight value = code * scale[row][col/16] * global.
 *
 * Memory and ownership:
 *   - Every pointer in nvfp4_moe_weights and nvfp4_moe_io is a DEVICE pointer
 *     owned by the caller. The handle BORROWS the weight pointers: they must stay
 *     valid until nvfp4_moe_destroy. The library allocates no device memory
 *     except what nvfp4_moe_create makes: a 256-byte status block and, when
 *     the layer can take the decode kernel, its state, kept zero between calls:
 *     the counters of its grid barrier, 256 bytes.
 *   - All other scratch lives in the caller's workspace (nvfp4_moe_workspace_bytes).
 *
 * Errors: every call returns 0 (NVFP4_MOE_OK) or a negative nvfp4_moe_status.
 *   Host-side checks run before anything is enqueued; a call that fails them
 *   enqueues nothing. Conditions found on the device (routing id out of range
 *   or duplicated, a non-finite routing logit, a non-finite computed value, a
 *   wait that gave up) are latched in the status block and returned by
 *   nvfp4_moe_get_status. forward never synchronises. Every device-side wait is
 *   bounded: a kernel whose wait runs out latches NVFP4_MOE_ERR_TIMEOUT and
 *   returns instead of hanging.
 *
 * Range: h = SiLU(g) * u is stored in F16 between the two projections, and the
 *   grouped-GEMM path (T > 8) stores each pair's w * s_d * y row in F16 before the
 *   FP32 combine. A value whose magnitude reaches 65520 there becomes inf; the
 *   layer then latches NVFP4_MOE_ERR_NONFINITE (detail: stage and expert) rather
 *   than return a silent inf. The tensor scales are applied in FP32 before these
 *   roundings, never folded into F16 operands, so ordinary scales stay well
 *   inside F16's normal range ("Strata NVFP4" README, "How it differs from
 *   upstream Strata": folding a tiny scale into FP16 activations pushed them
 *   into FP16 subnormals).
 *
 * Decode: calls with T <= 8 run one decode kernel (one CTA per SM) when its
 *   shared memory (the 8 activation rows at H, plus one CTA's slice of h) fits
 *   150 KB -- e.g. every layer with H <= 4096 and I <= 2048 at top-k <= 16 and
 *   <= 512 experts; other layers run small batches through the grouped-GEMM
 *   path. Each CTA computes gate/up, SwiGLU and the down projection for its own
 *   slice of the selected experts' intermediates; the slices' partial outputs are
 *   added as 64-bit integers (value x 2^32, rounded to nearest, so a partial sum
 *   must stay below 2^31 in magnitude, else the call reports
 *   NVFP4_MOE_ERR_NONFINITE): integer addition does not depend on the order of the
 *   adds, so, like the grouped-GEMM path, the decode kernel returns the same bits
 *   on every run. No CTA waits on another.
 *
 * Threading: a handle may be used from one host thread at a time. Two forward
 *   calls that run concurrently on the GPU must not share a workspace.
 */
#ifndef NVFP4_MOE_H
#define NVFP4_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NVFP4_MOE_ABI_VERSION 2
#define NVFP4_MOE_MAX_STACK 64   /* layers of one nvfp4_moe_forward_decode_stack call */

#if defined(__GNUC__)
#define NVFP4_MOE_API __attribute__((visibility("default")))
#else
#define NVFP4_MOE_API
#endif

/* Largest top-k the kernels support, the largest T the decode path takes, and
 * the largest max_tokens a handle accepts. */
#define NVFP4_MOE_MAX_TOPK 16
#define NVFP4_MOE_DECODE_MAX_T 8
#define NVFP4_MOE_MAX_TOKENS 65536

typedef enum {
    NVFP4_MOE_OK = 0,
    NVFP4_MOE_ERR_INVALID_ARG = -1,        /* null pointer, T<0, T>max_tokens, bad enum   */
    NVFP4_MOE_ERR_UNSUPPORTED_DIMS = -2,   /* H or I not a multiple of 32; K>E; K>16; E>1024;
                                              max_tokens > 65536                              */
    NVFP4_MOE_ERR_MISALIGNED = -3,         /* a plane or buffer not 16-byte aligned       */
    NVFP4_MOE_ERR_WORKSPACE_TOO_SMALL = -4,
    NVFP4_MOE_ERR_CUDA = -5,               /* a CUDA runtime/driver call failed           */
    NVFP4_MOE_ERR_BAD_ROUTING = -6,        /* device: precomputed id out of [0,E) or repeated */
    NVFP4_MOE_ERR_NONFINITE = -7,          /* device: a selected routing logit is NaN/inf, or a
                                              computed h, per-pair down row or output value is
                                              not finite (F16 intermediates overflowed)       */
    NVFP4_MOE_ERR_TIMEOUT = -8,            /* device: a bounded wait gave up              */
    NVFP4_MOE_ERR_NO_DEVICE = -9           /* no sm_100 device current                    */
} nvfp4_moe_status;

typedef struct nvfp4_moe nvfp4_moe_t; /* opaque handle */

/* Layer geometry. hidden = H, inter = I, n_experts = E, top_k = K.
 * max_tokens bounds T for every forward call and sizes the workspace.
 * H and I must be multiples of 32: whole groups of 16 inputs per scale ("TensorFold
 * PR #906", first post: cuts keep groups of 16) and code rows of a multiple of 16
 * bytes, which the tensor-map copies need. */
typedef struct {
    int32_t hidden;
    int32_t inter;
    int32_t n_experts;
    int32_t top_k;
    int32_t max_tokens;
} nvfp4_moe_dims;

/* Packed expert planes, DEVICE pointers, BORROWED (see above). Each code and
 * scale plane must be 16-byte aligned; the globals 4-byte aligned.
 *   gate_codes, up_codes   [E][I][H/2]  u8, two E2M1 codes per byte
 *   gate_scales, up_scales [E][I][H/16] E4M3 bytes, one per 16 inputs
 *   gate_global, up_global [E]          f32
 *   down_codes             [E][H][I/2]
 *   down_scales            [E][H][I/16]
 *   down_global            [E]                                            */
typedef struct {
    const uint8_t *gate_codes;
    const uint8_t *up_codes;
    const uint8_t *gate_scales;
    const uint8_t *up_scales;
    const float *gate_global;
    const float *up_global;
    const uint8_t *down_codes;
    const uint8_t *down_scales;
    const float *down_global;
} nvfp4_moe_weights;

typedef enum {
    NVFP4_MOE_ACT_BF16 = 0, /* act is [T][H] bf16                                 */
    NVFP4_MOE_ACT_INT8 = 1, /* act is [T][H] int8 q, x = q * act_scale[t] (f32)  */
    NVFP4_MOE_ACT_F32 = 2   /* act is [T][H] f32 (a residual stream); the layer's
                               input is its round-to-nearest-even BF16 value.
                               act may equal out with NVFP4_MOE_OUT_F32_ADD:
                               x <- x + layer(bf16(x)), one stacked-layer step.  */
} nvfp4_moe_act;

typedef enum {
    NVFP4_MOE_OUT_F32 = 0,     /* out[T][H] f32 = MoE(x)                          */
    NVFP4_MOE_OUT_F32_ADD = 1  /* out[T][H] f32 += MoE(x)  (residual stream)       */
} nvfp4_moe_out;

/* One forward call. DEVICE pointers, caller-owned.
 *   T               number of tokens, 0 <= T <= dims.max_tokens (T = 0 is a no-op)
 *   act, act_scale  activations; act_scale only for NVFP4_MOE_ACT_INT8
 *   router_logits   [T][E] f32; when NULL, either router_w projects the layer's
 *                   input to logits (below) or topk_ids [T][K] i32 and
 *                   topk_weights [T][K] f32 are used as given
 *   router_w        [E][H] bf16 router projection, or NULL. With router_logits
 *                   and topk_ids NULL, the library computes
 *                   logits[t][e] = sum_k router_w[e][k] * x[t][k] with x the
 *                   layer's input in FP32 -- never rounded to BF16 first: BF16
 *                   and FP32 activations as given, int8 ones as the FP32
 *                   product q * act_scale[t] -- and FP32 accumulation ("Strata
 *                   NVFP4" README, "How it differs from upstream Strata": the
 *                   router's BF16 projection takes FP32-exact inputs). Giving
 *                   router_w together with router_logits is INVALID_ARG;
 *                   router_w must be 16-byte aligned (else MISALIGNED).
 *   dbg_logits      optional (may be NULL) [T][E] f32: the computed router logits
 *   out             [T][H] f32, written (OUT_F32) or accumulated into (OUT_F32_ADD)
 *   dbg_*           optional (may be NULL) copies of the routing results:
 *                   dbg_ids [T][K] i32, dbg_w [T][K] f32 (renormalised weights),
 *                   dbg_counts [E] i32 (pairs per expert), dbg_offsets [E+1] i32
 *                   (exclusive scan of counts), dbg_perm [T*K] i32 (pair index
 *                   t*K+j, grouped by expert ascending, then token ascending).  */
typedef struct {
    int32_t T;
    nvfp4_moe_act act_type;
    const void *act;
    const float *act_scale;
    const float *router_logits;
    const int32_t *topk_ids;
    const float *topk_weights;
    nvfp4_moe_out out_type;
    float *out;
    int32_t *dbg_ids;
    float *dbg_w;
    int32_t *dbg_counts;
    int32_t *dbg_offsets;
    int32_t *dbg_perm;
    const uint16_t *router_w;   /* ABI version 2 */
    float *dbg_logits;          /* ABI version 2 */
} nvfp4_moe_io;

/* Validates dims and weight pointers (all checks before any allocation), then
 * allocates the handle, its device status block and decode state on the current
 * device. On failure *out is set to NULL and nothing stays allocated. Requires
 * an sm_100 device to be current.
 * Source: the pages' tensor readers validate the whole source before they
 * allocate, refuse incomplete or ambiguous scale data and free what they
 * allocated when an allocation fails ("TensorFold PR #906", first post); the
 * handle borrows the caller's planes instead of copying them ("#1858 ...
 * strata-safetensors", "Proposed contribution": bounded reads into buffers the
 * caller owns). */
NVFP4_MOE_API int nvfp4_moe_create(nvfp4_moe_t **out, const nvfp4_moe_dims *dims,
                     const nvfp4_moe_weights *weights);

/* Bytes of workspace a forward call with T tokens needs (256-byte aligned start
 * required). Returns 0 for a NULL handle or T outside [0, max_tokens].
 * Source: every buffer of a forward call is the caller's, sized up front ("#1858
 * ... strata-safetensors", "Proposed contribution": caller-owned bounded
 * buffers); the workspace holds the routing arrays, the per-pair activation and
 * h rows and the tile lists of the grouped GEMMs. */
NVFP4_MOE_API size_t nvfp4_moe_workspace_bytes(const nvfp4_moe_t *h, int32_t T);

/* Enqueues the whole layer on `stream` (a cudaStream_t; NULL = legacy default
 * stream). Asynchronous: never synchronises and never reads device memory back.
 * The workspace must not be used by another call until this one has finished
 * on the GPU. */
NVFP4_MOE_API int nvfp4_moe_forward(nvfp4_moe_t *h, const nvfp4_moe_io *io, void *workspace,
                      size_t workspace_bytes, void *stream);

/* Synchronises `stream`, returns the first device-side error latched since the
 * last call (0 if none) and clears it. After an error it also clears the decode
 * state a launch that gave up may have left behind.
 * Source: forward never waits on the host; the layer gathers each expert group
 * into one launch after one wait ("Strata NVFP4" README, "How it differs from
 * upstream Strata", the prompt-reading bullet), so device-side findings are
 * read once, here, instead of after every launch; what is refused (bad routing,
 * non-finite values) follows the readers' rule of refusing ambiguous or
 * incomplete data rather than guessing ("TensorFold PR #906", first post). */
NVFP4_MOE_API int nvfp4_moe_get_status(nvfp4_moe_t *h, void *stream);

/* Phase timing (optional): when n_events == NVFP4_MOE_PHASE_EVENTS and events
 * holds that many cudaEvent_t handles (created by the caller on the handle's
 * device), every later forward records event i on its stream at these phase
 * boundaries: 0 start, 1 routing done, 2 activation staging done, 3 gate/up +
 * SwiGLU done, 4 down + combine done. (Decode calls stage activations inside
 * routing, so events 1 and 2 coincide.) n_events == 0 turns it off. The handle
 * borrows the events; returns INVALID_ARG for any other n_events. This mirrors
 * per-phase accounting of a layer's time; it adds five event records per call.
 * The records are external (cudaEventRecordExternal), so a forward captured into
 * a CUDA graph records them on every replay. */
#define NVFP4_MOE_PHASE_EVENTS 5
NVFP4_MOE_API int nvfp4_moe_set_phase_events(nvfp4_moe_t *h, void *const *events, int32_t n_events);

/* Allocation-free decode call (the pages have no counterpart: this is a service
 * for callers that cannot allocate device memory at all, and so cannot create a
 * handle -- nvfp4_moe_create allocates a status block -- or pass a workspace).
 * It runs the same decode path as nvfp4_moe_forward for 1 <= T <= 8 tokens, with
 * its scratch in a 1 MiB array compiled into the library (a file-scope
 * __device__ array: every GPU that loads the library holds it until the process
 * exits). dims and weights are checked exactly as by nvfp4_moe_create; io and
 * stream are as for nvfp4_moe_forward. Calls no cudaMalloc/cudaFree.
 *   - T > 8, or a layer outside the decode kernel (see "Decode" above),
 *     returns NVFP4_MOE_ERR_UNSUPPORTED_DIMS; a layer whose decode scratch and
 *     state for this T exceed 1 MiB - 256 bytes would return
 *     NVFP4_MOE_ERR_WORKSPACE_TOO_SMALL (no layer the decode kernel takes needs
 *     that much: its state is 256 bytes and its shared memory bounds H and
 *     the expert count). Both are checked before anything is enqueued. T = 0
 *     is a no-op.
 *   - The first call on a device does a one-time set-up there: it looks up the
 *     array's device address (cudaGetSymbolAddress) and opts the decode kernels
 *     into the shared memory they need (cudaFuncSetAttribute). Make that first
 *     call before any stream capture on the device.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents; each call clears what must start at zero (the status words and
 *     the decode state, with one cudaMemsetAsync). Calls that overlap on
 *     the GPU (different streams, or other threads) race on it: serialise them.
 *   - Device-side routing problems (bad precomputed ids, non-finite logits) are
 *     contained exactly as in nvfp4_moe_forward but cannot be read back: there
 *     is no handle, hence no nvfp4_moe_get_status for this call. */
NVFP4_MOE_API int nvfp4_moe_forward_decode_static(const nvfp4_moe_dims *dims,
                                                  const nvfp4_moe_weights *weights,
                                                  const nvfp4_moe_io *io, void *stream);

/* Decode through a stack of layers in ONE kernel launch (T <= 8), over the FP32
 * residual stream: x <- x + layer_l(bf16(x)) for l = 0..n_layers-1, in place.
 * The pages measure the cost of launch gaps ("Strata NVFP4" README, "How it
 * differs from upstream Strata", the prompt-reading bullet: about 10 us idle
 * per wait); here the layers follow each other inside one kernel, separated by
 * grid barriers, with no launch between them.
 *   layers      n_layers handles (1 <= n_layers <= NVFP4_MOE_MAX_STACK) of
 *               identical dims on one device, each with max_tokens >= T; each
 *               layer's weights come from its handle; the status block and
 *               decode counters of layers[0] are used (read its get_status).
 *   io          act_type NVFP4_MOE_ACT_F32, out_type NVFP4_MOE_OUT_F32_ADD,
 *               act == out ([T][H] f32, updated in place); router_logits
 *               [n_layers][T][E] f32, layer l's at offset l*T*E; no router_w,
 *               no topk ids/weights, no dbg_* outputs (else INVALID_ARG).
 *   workspace   as for nvfp4_moe_forward on layers[0] with this T.
 * Returns UNSUPPORTED_DIMS when the layer does not take the decode kernel.
 * Every layer's arithmetic is that of nvfp4_moe_forward: the result equals
 * n_layers forward calls bit for bit. */
NVFP4_MOE_API int nvfp4_moe_forward_decode_stack(nvfp4_moe_t *const *layers, int32_t n_layers,
                                                 const nvfp4_moe_io *io, void *workspace,
                                                 size_t ws_bytes, void *stream);

/* Frees the handle, its status block and decode state. Never touches the
 * borrowed weights. */
NVFP4_MOE_API void nvfp4_moe_destroy(nvfp4_moe_t *h);

/* Static string for a status code. */
NVFP4_MOE_API const char *nvfp4_moe_strerror(int status);

/* ABI version compiled into the library (NVFP4_MOE_ABI_VERSION). */
NVFP4_MOE_API int nvfp4_moe_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_MOE_H */
