"""The allocation-free decode entry point, nvfp4_moe_forward_decode_static.

It serves callers that cannot allocate device memory at all: they can neither
create a handle (creation allocates a small status block) nor hand the layer a
workspace. This test calls it through the C ABI and requires its output to match
the regular entry point (handle + caller workspace) on the same inputs, within the
parity tolerance, for two calls in a row: the second call reuses the library's
static scratch, which still holds the first call's contents. It lives in a file of
its own that pytest collects last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
from helpers import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _io(nv, x, logits, out):
    return nv.IO(x.shape[0], nv.ACT_BF16, x.data_ptr(), None, logits.data_ptr(), None, None,
                 nv.OUT_F32, out.data_ptr(), None, None, None, None, None)


def test_static_decode_matches_regular_entry_point_twice():
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.LayerDims(E=64, H=512, I=384, K=6)
    layer = synth.make_layer(dims, seed=901).to(DEV)
    regular = nv.MoELayer.from_layer(layer, top_k=dims.K, max_tokens=8)
    cd = nv.Dims(dims.H, dims.I, dims.E, dims.K, 8)
    cw = nv.Weights(*[t.data_ptr() for t in layer.planes()])
    stream = torch.cuda.current_stream().cuda_stream
    for call, T in enumerate((8, 3)):
        x = synth.make_x_bf16(T, dims.H, seed=910 + call, outliers=True, device=DEV)
        logits = synth.make_logits(T, dims.E, seed=920 + call, zipf_s=1.1, device=DEV)
        want = regular.forward(x, logits=logits)
        got = torch.full((T, dims.H), float("nan"), dtype=torch.float32, device=DEV)
        rc = nv.nvfp4_moe_forward_decode_static(cd, cw, _io(nv, x, logits, got), stream)
        assert rc == 0, nv.nvfp4_moe_strerror(rc)
        torch.cuda.synchronize()
        assert_close(got.double().cpu().numpy(), want.double().cpu().numpy(),
                     f"static decode call {call + 1}")
    regular.close()


def test_static_decode_rejects_sizes_beyond_its_scratch():
    import nvfp4_mixture_experts_03_b200 as nv
    fake = nv.Weights(*[(1 << 40) + i * (1 << 30) for i in range(9)])
    x = torch.zeros(1, dtype=torch.uint8, device=DEV)
    big = nv.Dims(8192, 8192, 64, 16, 8)          # h alone needs 8*16*8192*2 B = 2 MiB
    io = nv.IO(8, nv.ACT_BF16, x.data_ptr(), None, x.data_ptr(), None, None, nv.OUT_F32,
               x.data_ptr(), None, None, None, None, None)
    assert nv.nvfp4_moe_forward_decode_static(big, fake, io, 0) == -4
    small = nv.Dims(256, 128, 8, 2, 16)
    io.T = 9                                          # beyond the decode path
    assert nv.nvfp4_moe_forward_decode_static(small, fake, io, 0) == -2
