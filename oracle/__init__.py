"""FP64 CPU oracle for the routed NVFP4 MoE layer -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import this package. The layer's CUDA path never does, and shares no code with it.

``liboracle.so`` is built from ``nvfp4_moe_oracle.c`` with the host C compiler
(``build()``); this module wraps it with ctypes and numpy.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_moe_oracle.c")
_HDR = os.path.join(_HERE, "nvfp4_moe_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

PLANT = {"none": 0, "nibble_order": 1, "group_shift": 2, "no_global": 3,
         "swap_gate_up": 4, "silu_sign": 5, "equal_weights": 6}


def build(force: bool = False) -> str:
    """Compile liboracle.so (plain C, -O2, no fast-math: IEEE FP64 throughout)."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC",
                               "-shared", "-std=c11", "-D_GNU_SOURCE", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class _Dims(C.Structure):
    _fields_ = [("E", C.c_int32), ("H", C.c_int32), ("I", C.c_int32), ("K", C.c_int32)]


class _Weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global", "up_global",
        "down_codes", "down_scales", "down_global")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.orc_e2m1.restype = C.c_double
        _lib.orc_e4m3.restype = C.c_double
        _lib.orc_bf16.restype = C.c_double
        _lib.orc_bf16.argtypes = [C.c_uint16]
        _lib.orc_bf16_rne.restype = C.c_uint16
        _lib.orc_bf16_rne.argtypes = [C.c_double]
        _lib.orc_route.restype = C.c_int
        _lib.orc_check_ids.restype = C.c_int
        _lib.orc_quantize.restype = C.c_int
        _lib.orc_moe.restype = C.c_int
        _lib.orc_pair_h.restype = C.c_int
        _lib.orc_pair_h.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_float,
                                    C.c_int32, C.c_void_p, C.c_int32]
        _lib.orc_router.argtypes = [C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                    C.c_void_p]
        _lib.orc_decode_matrix.argtypes = [C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                           C.c_float, C.c_void_p]
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return C.c_void_p(a.ctypes.data)


def _np(t):
    """torch tensor or numpy array -> contiguous numpy array on the host."""
    if hasattr(t, "detach"):
        t = t.detach().cpu()
        if str(t.dtype) == "torch.bfloat16":
            import torch
            t = t.view(torch.int16)
        t = t.contiguous().numpy()
    return np.ascontiguousarray(t)


def e2m1(nib: int) -> float:
    return lib().orc_e2m1(C.c_uint32(nib))


def e4m3(byte: int) -> float:
    return lib().orc_e4m3(C.c_uint32(byte))


def bf16(bits: int) -> float:
    return lib().orc_bf16(C.c_uint16(bits))


def bf16_rne(v: float) -> int:
    return lib().orc_bf16_rne(C.c_double(v))


def bf16_rne_array(v) -> np.ndarray:
    """FP64 array -> BF16 bits (uint16), each the nearest BF16, ties to even."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    out = np.zeros(a.shape, np.uint16)
    lib().orc_bf16_rne_array(C.c_int64(a.size), _p(a), _p(out))
    return out


def route(logits, K: int):
    """-> (ids int32 [T][K], w float64 [T][K], n_nonfinite_tokens)"""
    l = _np(logits).astype(np.float32, copy=False)
    T, E = l.shape
    ids = np.zeros((T, K), np.int32)
    w = np.zeros((T, K), np.float64)
    bad = lib().orc_route(C.c_int32(T), C.c_int32(E), C.c_int32(K), _p(l), _p(ids), _p(w))
    return ids, w, bad


def router_input(x, x_scale=None) -> np.ndarray:
    """The router's FP32 input for the layer's activations: BF16 and FP32 values
    as they are (exact in FP32); int8 codes as the FP32 product q * scale (one
    correctly rounded multiply), which is what a reader of the scaled
    activations holds."""
    a = _np(x)
    if a.dtype == np.int16:   # BF16 bits
        return (a.astype(np.uint16).astype(np.uint32) << 16).view(np.float32)
    if a.dtype == np.int8:
        s = _np(x_scale).astype(np.float32)
        return a.astype(np.float32) * s[:, None]
    return a.astype(np.float32, copy=False)


def router(x_f32, w_r_bf16) -> np.ndarray:
    """FP64 router logits [T][E] = W_r x for FP32 x [T][H] and BF16 W_r [E][H]."""
    x = np.ascontiguousarray(_np(x_f32).astype(np.float32, copy=False))
    w = np.ascontiguousarray(_np(w_r_bf16).astype(np.uint16, copy=False))
    T, H = x.shape
    E = w.shape[0]
    assert w.shape[1] == H
    out = np.zeros((T, E), np.float64)
    lib().orc_router(C.c_int32(T), C.c_int32(E), C.c_int32(H), _p(x), _p(w), _p(out))
    return out


def check_ids(ids, E: int) -> int:
    i = _np(ids).astype(np.int32, copy=False)
    T, K = i.shape
    return lib().orc_check_ids(C.c_int32(T), C.c_int32(E), C.c_int32(K), _p(i))


def sort(ids, E: int):
    """-> (counts [E], offsets [E+1], perm [T*K]) int32"""
    i = _np(ids).astype(np.int32, copy=False)
    T, K = i.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * K, np.int32)
    lib().orc_sort(C.c_int32(T), C.c_int32(E), C.c_int32(K), _p(i), _p(counts), _p(offsets),
                   _p(perm))
    return counts, offsets, perm


def quantize(w_bf16):
    """BF16 weights [n][rows][cols] (torch bf16 or uint16/int16 bits) ->
    (codes u8 [n][rows][cols/2], scales u8 [n][rows][cols/16], glob f32 [n])."""
    w = _np(w_bf16).view(np.uint16)
    if w.ndim == 2:
        w = w[None]
    n, rows, cols = w.shape
    codes = np.zeros((n, rows, cols // 2), np.uint8)
    scales = np.zeros((n, rows, cols // 16), np.uint8)
    glob = np.zeros(n, np.float32)
    rc = lib().orc_quantize(C.c_int32(n), C.c_int32(rows), C.c_int32(cols), _p(w), _p(codes),
                            _p(scales), _p(glob))
    assert rc == 0
    return codes, scales, glob


def decode_matrix(codes, scales, glob) -> np.ndarray:
    c, s = _np(codes), _np(scales)
    rows, cols = c.shape[0], c.shape[1] * 2
    out = np.zeros((rows, cols), np.float64)
    lib().orc_decode_matrix(C.c_int32(rows), C.c_int32(cols), _p(c), _p(s), C.c_float(float(glob)),
                            _p(out))
    return out


def quantize_act_nvfp4(x_bf16):
    """Activations as an FP4 x FP4 prompt path multiplies them ("Strata NVFP4"
    README, "How it differs from upstream Strata", the W4A8 bullet: llama.cpp's
    NVFP4 prompt path on sm_120 runs FP4 x FP4). The pages do not print the
    activation recipe; the reading taken is the checkpoint's own NVFP4 recipe
    applied per token: each token row is one tensor for `quantize` (global =
    amax / (6 * 448) in FP32, an E4M3 scale per 16 elements, E2M1 codes nearest).
    x: BF16 [T][H] (torch bf16 or uint16 bits) ->
    (codes u8 [T][H/2], scales u8 [T][H/16], glob f32 [T])."""
    x = _np(x_bf16).view(np.uint16)
    codes, scales, glob = quantize(np.ascontiguousarray(x[:, None, :]))
    return codes[:, 0], scales[:, 0], glob


def dequant_act_nvfp4(codes, scales, glob) -> np.ndarray:
    """FP64 [T][H] values of per-token NVFP4 activations (each row decoded with
    its own global)."""
    return np.concatenate([decode_matrix(codes[t:t + 1], scales[t:t + 1], glob[t])
                           for t in range(len(glob))])


def quantize_act_int8(x_bf16):
    """Per-token symmetric int8, the activation format of the W4A8 prompt path
    ("Strata NVFP4" README, "How it differs from upstream Strata", the W4A8 bullet:
    8-bit activations), as this layer takes it: scale_t = amax_t / 127 rounded to
    FP32, q = nearest integer of x / scale_t (ties to even), clamped to +-127.
    -> (q int8 [T][H], scale f32 [T])."""
    x = _np(x_bf16).view(np.uint16)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    scale = (np.abs(xf).max(axis=1) / 127.0).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float64)
    q = np.clip(np.rint(xf / safe[:, None]), -127, 127).astype(np.int8)
    return q, scale


F16_MAX = 65504.0


def quantize_h_int8_blocks(h, block: int = 32):
    """8-bit h for the down projection as a fused SwiGLU quantiser makes it
    ("Strata NVFP4" README, the 0.1.39-nvfp4.2 bullet: the quantiser keeps its FP16
    scale finite). Reading taken: blocks of `block` consecutive intermediates, an
    FP16 scale d = amax / 127 rounded to nearest FP16 and clamped to the largest
    finite FP16 value, q = nearest integer of h / d (ties to even) clamped to
    +-127; a zero block has d = 0 and q = 0.
    h: FP64 [n][I] -> (q int8 [n][I], d f16 [n][I/block])."""
    h = np.asarray(h, np.float64)
    n, I = h.shape
    hb = h.reshape(n, I // block, block)
    d = np.minimum(np.abs(hb).max(axis=2) / 127.0, F16_MAX).astype(np.float16)
    d64 = d.astype(np.float64)
    safe = np.where(d64 > 0, d64, 1.0)
    q = np.clip(np.rint(hb / safe[:, :, None]), -127, 127)
    q = np.where(d64[:, :, None] > 0, q, 0).astype(np.int8)
    return q.reshape(n, I), d


def dequant_h_int8_blocks(q, d, block: int = 32) -> np.ndarray:
    n, I = q.shape
    return (q.astype(np.float64).reshape(n, I // block, block) *
            d.astype(np.float64)[:, :, None]).reshape(n, I)


def quantize_h_int8_rows(h):
    """Per-row int8 h: scale = amax / 127 in FP32, q = nearest integer of h / scale
    (ties to even) clamped to +-127. -> (q int8 [n][I], scale f32 [n])."""
    h = np.asarray(h, np.float64)
    s = (np.abs(h).max(axis=1) / 127.0).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float64)
    return np.clip(np.rint(h / safe[:, None]), -127, 127).astype(np.int8), s


_E4M3_POS = None


def quantize_h_e4m3_rows(h):
    """Per-row FP8 h: scale = amax / 448 in FP32 (the row's largest value maps to
    E4M3's largest finite value), each h / scale rounded to the nearest E4M3 value
    (ties to the even code), searched over the decoded table of all finite
    bytes. -> (codes u8 [n][I], scale f32 [n])."""
    global _E4M3_POS
    if _E4M3_POS is None:
        _E4M3_POS = np.array([e4m3(b) for b in range(127)])     # bytes 0x00..0x7E
    h = np.asarray(h, np.float64)
    s = (np.abs(h).max(axis=1) / 448.0).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float64)
    r = np.abs(h) / safe[:, None]
    dist = np.abs(r[..., None] - _E4M3_POS)
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    # ties: the even byte (a table step is one code apart, so of two equally near
    # neighbours exactly one is even)
    even = (np.arange(127) % 2 == 0)
    pick = np.where(cand.sum(axis=-1) > 1, np.argmax(cand & even, axis=-1), np.argmax(cand, axis=-1))
    codes = pick.astype(np.uint8) | np.where(h < 0, 0x80, 0).astype(np.uint8)
    return codes, s


def dequant_h_e4m3_rows(codes, s) -> np.ndarray:
    mag = np.array([e4m3(b) for b in range(128)])[codes & 0x7F]
    return np.where(codes & 0x80, -mag, mag) * s.astype(np.float64)[:, None]


def layer_with_h(layer, x, ids, wts, *, K: int, sample, h_rounds=(None,)) -> list:
    """Layer outputs, FP64 [n][H] each, for the tokens in `sample`, one per entry of
    `h_rounds`: each pair's h (the oracle's, FP64) goes through that callable
    ([n][I] -> [n][I]; None keeps it) before the down projection:
    out_t = sum_j w_tj * D_e (h_round(h_tj)), D_e decoded with its global. The h
    of every pair is computed once for all entries; the None entry is `moe`'s
    result."""
    xa = _np(x)
    ia = _np(ids).astype(np.int32)
    wa = _np(wts).astype(np.float64)
    dc, ds, dg = (_np(layer.down_codes), _np(layer.down_scales), _np(layer.down_global))
    D = {}
    outs = [np.zeros((len(sample), dc.shape[1])) for _ in h_rounds]
    for n, t in enumerate(sample):
        hs = np.stack([pair_h(layer, xa[t], int(e), K=K) for e in ia[t]])
        for out, f in zip(outs, h_rounds):
            hq = hs if f is None else f(hs)
            for j, e in enumerate(ia[t]):
                e = int(e)
                if e not in D:
                    D[e] = decode_matrix(dc[e], ds[e], dg[e])
                out[n] += wa[t, j] * (D[e] @ hq[j])
    return outs


class _Bound:
    """ctypes views of one layer's planes (keeps the numpy arrays alive)."""

    def __init__(self, layer, K: int):
        self.arrs = {k: _np(getattr(layer, k)) for k in (
            "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global", "up_global",
            "down_codes", "down_scales", "down_global")}
        E, I, H2 = self.arrs["gate_codes"].shape
        self.dims = _Dims(E, H2 * 2, I, K)
        self.w = _Weights(**{k: v.ctypes.data for k, v in self.arrs.items()})


def moe(layer, x, ids, wts, *, K: int, x_scale=None, sample=None, nthreads: int = 0,
        plant: str | int = 0) -> np.ndarray:
    """Layer output, FP64 [n][H], for the tokens in `sample` (all when None).
    x: BF16 [T][H] (torch bf16 or uint16 bits) or int8 [T][H] with x_scale [T]."""
    b = _Bound(layer, K)
    xa = _np(x)
    act_type = 1 if xa.dtype == np.int8 else 0
    if act_type == 0:
        xa = xa.view(np.uint16)
    T = xa.shape[0]
    xs = _np(x_scale).astype(np.float32) if x_scale is not None else np.zeros(1, np.float32)
    ia = _np(ids).astype(np.int32)
    wa = _np(wts).astype(np.float64)
    samp = None if sample is None else np.ascontiguousarray(np.asarray(sample, np.int32))
    n = T if samp is None else len(samp)
    out = np.zeros((n, b.dims.H), np.float64)
    pl = PLANT[plant] if isinstance(plant, str) else int(plant)
    rc = lib().orc_moe(C.byref(b.dims), C.byref(b.w), C.c_int32(T), C.c_int32(act_type), _p(xa),
                       _p(xs), _p(ia), _p(wa), C.c_int32(n),
                       _p(samp) if samp is not None else None, _p(out), C.c_int32(nthreads),
                       C.c_int32(pl))
    assert rc == 0, "oracle rejected its arguments"
    return out


def pair_h(layer, x_row, e: int, *, K: int, x_scale: float = 1.0, plant=0) -> np.ndarray:
    b = _Bound(layer, K)
    xa = _np(x_row)
    act_type = 1 if xa.dtype == np.int8 else 0
    if act_type == 0:
        xa = xa.view(np.uint16)
    h = np.zeros(b.dims.I, np.float64)
    pl = PLANT[plant] if isinstance(plant, str) else int(plant)
    lib().orc_pair_h(C.byref(b.dims), C.byref(b.w), act_type, _p(np.ascontiguousarray(xa)),
                     x_scale, e, _p(h), pl)
    return h


def forward(layer, x, *, K: int, logits=None, ids=None, wts=None, x_scale=None, sample=None,
            nthreads: int = 0, plant=0, router_w=None):
    """Route (or take ids/weights as given) and run the layer. With `router_w`
    (BF16 [E][H]) the logits are the router projection of the layer's input,
    rounded to FP32 for the selection.
    -> dict(out, ids, w, counts, offsets, perm, nonfinite[, logits64])"""
    E = _np(layer.gate_global).shape[0]
    logits64 = None
    if router_w is not None:
        logits64 = router(router_input(x, x_scale), router_w)
        logits = logits64.astype(np.float32)
    if _np(x).dtype == np.float32:
        # FP32 activations (a residual stream): the experts take their nearest
        # BF16 values, ties to even
        x = bf16_rne_array(_np(x).astype(np.float64))
    if logits is not None:
        ids, w, bad = route(logits, K)
    else:
        ids = _np(ids).astype(np.int32)
        w = _np(wts).astype(np.float64)
        bad = 0
    counts, offsets, perm = sort(ids, E)
    out = moe(layer, x, ids, w, K=K, x_scale=x_scale, sample=sample, nthreads=nthreads,
              plant=plant)
    res = dict(out=out, ids=ids, w=w, counts=counts, offsets=offsets, perm=perm, nonfinite=bad)
    if logits64 is not None:
        res["logits64"] = logits64
    return res
