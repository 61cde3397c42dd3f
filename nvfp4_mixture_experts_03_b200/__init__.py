"""Python binding of the NVFP4 MoE layer's C ABI (include/nvfp4_moe.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libnvfp4_moe.so``. PyTorch is used for device memory and streams. There is no
CPU fallback: importing works without a GPU, but every call that needs the
library raises if it is missing or was not built.

Low-level names mirror the C ABI (``nvfp4_moe_create``, ``nvfp4_moe_forward``,
...). ``MoELayer`` wraps one handle together with the tensors it borrows.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4_moe.so")

OK = 0
ERR = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED_DIMS", -3: "MISALIGNED",
       -4: "WORKSPACE_TOO_SMALL", -5: "CUDA", -6: "BAD_ROUTING", -7: "NONFINITE",
       -8: "TIMEOUT", -9: "NO_DEVICE"}
ACT_BF16, ACT_INT8, ACT_F32 = 0, 1, 2
OUT_F32, OUT_F32_ADD = 0, 1
DECODE_MAX_T = 8
MAX_TOPK = 16

# Every function the headers declare (checked against include/*.h by the tests).
EXPORTS = ("nvfp4_moe_create", "nvfp4_moe_workspace_bytes", "nvfp4_moe_forward",
           "nvfp4_moe_get_status", "nvfp4_moe_destroy", "nvfp4_moe_strerror",
           "nvfp4_moe_abi_version", "nvfp4_moe_set_phase_events",
           "nvfp4_moe_forward_decode_static", "nvfp4_moe_forward_decode_stack",
           "nvfp4_moe_test_set_flags", "nvfp4_moe_test_fail_alloc", "nvfp4_moe_test_last_detail")
TEST_DECODE_STALL = 1   # include/nvfp4_moe_test.h
TEST_NO_SMALL = 2       # every used expert takes the grouped-GEMM tiles
PHASE_EVENTS = 5


class Dims(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("max_tokens", C.c_int32)]


class Weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global", "up_global",
        "down_codes", "down_scales", "down_global")]


class IO(C.Structure):
    _fields_ = [("T", C.c_int32), ("act_type", C.c_int), ("act", C.c_void_p),
                ("act_scale", C.c_void_p), ("router_logits", C.c_void_p),
                ("topk_ids", C.c_void_p), ("topk_weights", C.c_void_p),
                ("out_type", C.c_int), ("out", C.c_void_p), ("dbg_ids", C.c_void_p),
                ("dbg_w", C.c_void_p), ("dbg_counts", C.c_void_p), ("dbg_offsets", C.c_void_p),
                ("dbg_perm", C.c_void_p), ("router_w", C.c_void_p), ("dbg_logits", C.c_void_p)]


class NVFP4MoEError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {ERR.get(code, code)} ({nvfp4_moe_strerror(code)})")


_lib = None


def lib() -> C.CDLL:
    """The loaded CUDA library. Raises if it was not built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run __graft_entry__.build() or "
                               "python -m nvfp4_mixture_experts_03_b200.build")
        L = C.CDLL(LIB_PATH)
        L.nvfp4_moe_create.restype = C.c_int
        L.nvfp4_moe_create.argtypes = [C.POINTER(C.c_void_p), C.POINTER(Dims), C.POINTER(Weights)]
        L.nvfp4_moe_workspace_bytes.restype = C.c_size_t
        L.nvfp4_moe_workspace_bytes.argtypes = [C.c_void_p, C.c_int32]
        L.nvfp4_moe_forward.restype = C.c_int
        L.nvfp4_moe_forward.argtypes = [C.c_void_p, C.POINTER(IO), C.c_void_p, C.c_size_t,
                                        C.c_void_p]
        L.nvfp4_moe_get_status.restype = C.c_int
        L.nvfp4_moe_get_status.argtypes = [C.c_void_p, C.c_void_p]
        L.nvfp4_moe_destroy.restype = None
        L.nvfp4_moe_destroy.argtypes = [C.c_void_p]
        L.nvfp4_moe_strerror.restype = C.c_char_p
        L.nvfp4_moe_strerror.argtypes = [C.c_int]
        L.nvfp4_moe_abi_version.restype = C.c_int
        L.nvfp4_moe_set_phase_events.restype = C.c_int
        L.nvfp4_moe_set_phase_events.argtypes = [C.c_void_p, C.POINTER(C.c_void_p), C.c_int32]
        L.nvfp4_moe_test_last_detail.restype = C.c_int
        L.nvfp4_moe_test_last_detail.argtypes = [C.c_void_p]
        L.nvfp4_moe_forward_decode_stack.restype = C.c_int
        L.nvfp4_moe_forward_decode_stack.argtypes = [C.POINTER(C.c_void_p), C.c_int32, C.POINTER(IO),
                                                     C.c_void_p, C.c_size_t, C.c_void_p]
        L.nvfp4_moe_forward_decode_static.restype = C.c_int
        L.nvfp4_moe_forward_decode_static.argtypes = [C.POINTER(Dims), C.POINTER(Weights),
                                                      C.POINTER(IO), C.c_void_p]
        _lib = L
    return _lib


# ----------------------------------------------------------- C ABI, 1:1

def nvfp4_moe_create(dims: Dims, weights: Weights) -> int:
    h = C.c_void_p()
    rc = lib().nvfp4_moe_create(C.byref(h), C.byref(dims), C.byref(weights))
    if rc != OK:
        raise NVFP4MoEError(rc, "nvfp4_moe_create")
    return h.value


def nvfp4_moe_workspace_bytes(handle: int, T: int) -> int:
    return lib().nvfp4_moe_workspace_bytes(C.c_void_p(handle), T)


def nvfp4_moe_forward(handle: int, io: IO, workspace: int, workspace_bytes: int, stream: int) -> int:
    return lib().nvfp4_moe_forward(C.c_void_p(handle), C.byref(io), C.c_void_p(workspace),
                                   workspace_bytes, C.c_void_p(stream))


def nvfp4_moe_get_status(handle: int, stream: int) -> int:
    return lib().nvfp4_moe_get_status(C.c_void_p(handle), C.c_void_p(stream))


def nvfp4_moe_destroy(handle: int) -> None:
    lib().nvfp4_moe_destroy(C.c_void_p(handle))


def nvfp4_moe_strerror(code: int) -> str:
    try:
        return lib().nvfp4_moe_strerror(code).decode()
    except RuntimeError:
        return ERR.get(code, "unknown")


def nvfp4_moe_abi_version() -> int:
    return lib().nvfp4_moe_abi_version()


def nvfp4_moe_set_phase_events(handle: int, events) -> int:
    """events: sequence of PHASE_EVENTS cudaEvent_t handles (ints), or () to turn off."""
    arr = (C.c_void_p * max(1, len(events)))(*[C.c_void_p(int(e)) for e in events])
    return lib().nvfp4_moe_set_phase_events(C.c_void_p(handle), arr, len(events))


def nvfp4_moe_test_set_flags(handle: int, flags: int) -> int:
    """Test hook (include/nvfp4_moe_test.h): TEST_DECODE_STALL makes decode's grid
    barrier wait run out, so the call latches TIMEOUT; TEST_NO_SMALL sends every
    used expert through the grouped-GEMM tiles (none through the small-expert
    kernels)."""
    return lib().nvfp4_moe_test_set_flags(C.c_void_p(handle), C.c_int32(flags))


def nvfp4_moe_test_last_detail(handle: int) -> int:
    """Test hook: the detail word of the status the last get_status returned."""
    return lib().nvfp4_moe_test_last_detail(C.c_void_p(handle))


def nvfp4_moe_test_fail_alloc(n: int) -> None:
    """Test hook: the n-th device allocation of later creates fails (then disarms)."""
    lib().nvfp4_moe_test_fail_alloc(C.c_int32(n))


def nvfp4_moe_forward_decode_stack(handles, io: IO, workspace: int, ws_bytes: int, stream: int) -> int:
    """One launch for a stack of decode layers over the FP32 residual stream."""
    arr = (C.c_void_p * len(handles))(*handles)
    return lib().nvfp4_moe_forward_decode_stack(arr, len(handles), C.byref(io), C.c_void_p(workspace),
                                                C.c_size_t(ws_bytes), C.c_void_p(stream))


def decode_stack(layers, x, logits, *, workspace=None, stream=None):
    """x <- x + layer_l(bf16(x)) for every MoELayer in `layers`, in place, in one
    kernel launch. x: [T][H] f32 (T <= 8); logits: [L][T][E] f32. Returns x."""
    T = x.shape[0]
    ws = workspace if workspace is not None else layers[0].workspace(T)
    act_type = {torch.bfloat16: ACT_BF16, torch.int8: ACT_INT8, torch.float32: ACT_F32}[x.dtype]
    io = IO(T, act_type, _ptr(x), None, _ptr(logits), None, None, OUT_F32_ADD, _ptr(x),
            None, None, None, None, None, None, None)
    rc = nvfp4_moe_forward_decode_stack([m.handle for m in layers], io, ws.data_ptr(), ws.numel(),
                                        _stream_handle(stream))
    if rc != OK:
        raise NVFP4MoEError(rc, "nvfp4_moe_forward_decode_stack")
    return x


def nvfp4_moe_forward_decode_static(dims: Dims, weights: Weights, io: IO, stream: int) -> int:
    """Allocation-free decode (T <= 8): scratch is a 1 MiB array inside the library,
    shared by every call on the device -- serialise calls. No handle, no workspace."""
    return lib().nvfp4_moe_forward_decode_static(C.byref(dims), C.byref(weights), C.byref(io),
                                                 C.c_void_p(stream))


# ------------------------------------------------------------ torch glue

def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class MoELayer:
    """One layer's handle plus the device tensors it borrows.

    planes: (gate_codes, up_codes, gate_scales, up_scales, gate_global, up_global,
    down_codes, down_scales, down_global), contiguous CUDA tensors in the header's
    layouts.
    """

    def __init__(self, planes, *, top_k: int, max_tokens: int):
        planes = tuple(planes)
        for t in planes:
            if not (t.is_cuda and t.is_contiguous()):
                raise ValueError("weight planes must be contiguous CUDA tensors")
        self.planes = planes  # keeps the borrowed memory alive
        gc = planes[0]
        E, I, H2 = gc.shape
        self.E, self.I, self.H, self.K = E, I, 2 * H2, top_k
        self.max_tokens = max_tokens
        self.dims = Dims(self.H, self.I, E, top_k, max_tokens)
        self.weights = Weights(*[t.data_ptr() for t in planes])
        with torch.cuda.device(gc.device):
            self.handle = nvfp4_moe_create(self.dims, self.weights)
        self.device = gc.device
        self._ws = None

    @classmethod
    def from_layer(cls, layer, *, top_k: int, max_tokens: int):
        return cls(layer.planes(), top_k=top_k, max_tokens=max_tokens)

    def workspace_bytes(self, T: int) -> int:
        return nvfp4_moe_workspace_bytes(self.handle, T)

    def workspace(self, T: int) -> torch.Tensor:
        n = self.workspace_bytes(T)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def forward(self, x, *, logits=None, topk_ids=None, topk_weights=None, x_scale=None,
                out=None, accumulate: bool = False, debug: dict | None = None,
                workspace=None, stream=None, router_w=None) -> torch.Tensor:
        """Enqueue the layer on `stream` (default: torch's current stream).
        x: [T][H] bf16, int8 (with x_scale [T] f32) or f32 (residual stream).
        Routing from `logits` [T][E] f32, from the router projection `router_w`
        [E][H] bf16 of x, or from `topk_ids`/`topk_weights` as given.
        Returns `out` ([T][H] f32)."""
        T = x.shape[0]
        act_type = {torch.bfloat16: ACT_BF16, torch.int8: ACT_INT8, torch.float32: ACT_F32}[x.dtype]
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.float32, device=x.device)
        dbg = debug if debug is not None else {}
        io = IO(T, act_type, _ptr(x), _ptr(x_scale), _ptr(logits), _ptr(topk_ids),
                _ptr(topk_weights), OUT_F32_ADD if accumulate else OUT_F32, _ptr(out),
                _ptr(dbg.get("ids")), _ptr(dbg.get("w")), _ptr(dbg.get("counts")),
                _ptr(dbg.get("offsets")), _ptr(dbg.get("perm")), _ptr(router_w),
                _ptr(dbg.get("logits")))
        ws = workspace if workspace is not None else self.workspace(T)
        rc = nvfp4_moe_forward(self.handle, io, ws.data_ptr(), ws.numel(), _stream_handle(stream))
        if rc != OK:
            raise NVFP4MoEError(rc, "nvfp4_moe_forward")
        return out

    def set_phase_events(self, events):
        """events: PHASE_EVENTS torch.cuda.Event(enable_timing=True) objects, or ().
        The events are recorded at the phase boundaries of every later forward."""
        for ev in events:
            if ev.cuda_event == 0:
                ev.record()  # materialise the underlying cudaEvent_t
        self._phase_events = tuple(events)
        rc = nvfp4_moe_set_phase_events(self.handle, [ev.cuda_event for ev in events])
        if rc != OK:
            raise NVFP4MoEError(rc, "nvfp4_moe_set_phase_events")

    def status(self, stream=None) -> int:
        return nvfp4_moe_get_status(self.handle, _stream_handle(stream))

    def close(self):
        if getattr(self, "handle", None):
            nvfp4_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def debug_buffers(T: int, E: int, K: int, device) -> dict:
    """Optional routing outputs for checks: ids, w, counts, offsets, perm, and the
    router projection's logits (written only when the layer computes them)."""
    i32 = dict(dtype=torch.int32, device=device)
    return {"ids": torch.empty(T, K, **i32), "w": torch.empty(T, K, dtype=torch.float32, device=device),
            "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
            "perm": torch.empty(T * K, **i32),
            "logits": torch.empty(T, E, dtype=torch.float32, device=device)}
