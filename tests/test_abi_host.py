"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/nvfp4_moe.h declares, and rejects bad arguments before it
touches the device."""
import ctypes as C
import os
import re

import pytest

import nvfp4_mixture_experts_03_b200 as nv
from conftest import ROOT

HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(nvfp4_moe_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    from nvfp4_mixture_experts_03_b200 import build
    build.build()
    return nv.lib()


def test_header_declares_the_abi():
    assert declared_functions() == sorted(nv.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert nv.nvfp4_moe_abi_version() == 2
    for code in nv.ERR:
        assert nv.nvfp4_moe_strerror(code) not in ("", "unknown status")
    assert nv.nvfp4_moe_strerror(12345) == "unknown status"


def _weights(align=256):
    # fake (never dereferenced) device addresses; create rejects before using them
    base = 1 << 40
    return nv.Weights(*[base + i * (1 << 30) + (align if align != 256 else 0) for i in range(9)])


@pytest.mark.parametrize("dims,code", [
    ((2048, 768, 512, 10, 64), None),            # valid dims: fails later (no device / fake ptrs)
    ((2080, 800, 512, 10, 64), None),            # H, I multiples of 32 (not of 128): valid
    ((2048, 700, 512, 10, 64), -2),              # I not a multiple of 32
    ((2000, 768, 512, 10, 64), -2),              # H not a multiple of 32
    ((2048, 768, 8, 10, 64), -2),                # K > E
    ((2048, 768, 512, 17, 64), -2),              # K > 16
    ((2048, 768, 2048, 10, 64), -2),             # E > 1024
    ((2048, 768, 512, 0, 64), -1),               # K = 0
    ((2048, 768, 512, 10, -1), -1),              # negative max_tokens
    ((2048, 768, 512, 10, 65537), -2),           # max_tokens above the routing scan's limit
])
def test_create_validates_dims_before_device(L, dims, code):
    h = C.c_void_p(123)
    rc = L.nvfp4_moe_create(C.byref(h), C.byref(nv.Dims(*dims)), C.byref(_weights()))
    if code is None:
        assert rc in (-9, -5, 0)
        if rc == 0:
            L.nvfp4_moe_destroy(h)
    else:
        assert rc == code
    if rc != 0:
        assert h.value is None  # *out cleared on failure


def test_create_rejects_null_and_misaligned_planes(L):
    d = nv.Dims(256, 128, 8, 2, 64)
    w = _weights()
    w.down_scales = None
    h = C.c_void_p()
    assert L.nvfp4_moe_create(C.byref(h), C.byref(d), C.byref(w)) == -1
    w = _weights()
    w.up_codes = (1 << 40) + 8
    assert L.nvfp4_moe_create(C.byref(h), C.byref(d), C.byref(w)) == -3
    assert L.nvfp4_moe_create(None, C.byref(d), C.byref(w)) == -1


def test_forward_and_status_reject_null_handle(L):
    io = nv.IO()
    assert L.nvfp4_moe_forward(None, C.byref(io), None, 0, None) == -1
    assert L.nvfp4_moe_get_status(None, None) == -1
    assert L.nvfp4_moe_workspace_bytes(None, 4) == 0
    L.nvfp4_moe_destroy(None)   # no-op
