"""Fault paths on the GPU, driven by the test hooks of include/nvfp4_moe_test.h
and by host-side changes. No test here faults, traps or hangs a GPU: the stall
test makes the decode kernel's bounded grid-barrier wait run out (about 200 ms)
and checks that the call reports TIMEOUT and that the handle is correct again
afterwards; the overflow test makes the layer's own arithmetic overflow (scaled
global scales, swapped in place under a live handle); the allocation test makes
create's device allocations fail one at a time."""
import pytest

import oracle
import synth
from helpers import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"
NONFINITE, TIMEOUT, CUDA_ERR, INVALID = -7, -8, -5, -1


def _layer():
    dims = synth.LayerDims(E=16, H=256, I=256, K=4)
    return dims, synth.make_layer(dims, seed=61)


def test_decode_wait_runs_out_then_recovers():
    import nvfp4_mixture_experts_03_b200 as nv
    dims, layer = _layer()
    T = 3
    x = synth.make_x_bf16(T, dims.H, 62)
    logits = synth.make_logits(T, dims.E, 62)
    ref = oracle.forward(layer, x, K=dims.K, logits=logits)
    m = nv.MoELayer.from_layer(layer.to(DEV), top_k=dims.K, max_tokens=8)
    try:
        assert nv.nvfp4_moe_test_set_flags(m.handle, nv.TEST_DECODE_STALL) == 0
        m.forward(x.to(DEV), logits=logits.to(DEV))
        assert m.status() == TIMEOUT
        assert nv.nvfp4_moe_test_set_flags(m.handle, 0) == 0
        for _ in range(2):   # the state left by the stalled call was cleared by status()
            out = m.forward(x.to(DEV), logits=logits.to(DEV))
            assert m.status() == 0
            assert_close(out.double().cpu().numpy(), ref["out"], "decode after a timeout")
        assert nv.nvfp4_moe_test_set_flags(m.handle, 8) == INVALID   # unknown flag
    finally:
        m.close()


@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_decode_recovers_after_nonfinite(which):
    """gate and up x 2^12 push h past F16; an infinite down scale makes the output
    non-finite. Either way the call must report NONFINITE, and the next calls on the
    same handle (globals restored) must match the oracle: nothing of the failed
    call's state survives."""
    import nvfp4_mixture_experts_03_b200 as nv
    dims, layer = _layer()
    T = 3
    x = synth.make_x_bf16(T, dims.H, 62)
    logits = synth.make_logits(T, dims.E, 62)
    ref = oracle.forward(layer, x, K=dims.K, logits=logits)
    dl = layer.to(DEV)
    m = nv.MoELayer.from_layer(dl, top_k=dims.K, max_tokens=8)
    try:
        gs = [dl.gate_global, dl.up_global] if which == "gate_up" else [dl.down_global]
        keep = [g.clone() for g in gs]
        for g in gs:
            if which == "gate_up":
                g.mul_(2.0 ** 12)
            else:
                g.fill_(float("inf"))
        m.forward(x.to(DEV), logits=logits.to(DEV))
        assert m.status() == NONFINITE
        for g, k in zip(gs, keep):
            g.copy_(k)
        for _ in range(2):
            out = m.forward(x.to(DEV), logits=logits.to(DEV))
            assert m.status() == 0
            assert_close(out.double().cpu().numpy(), ref["out"], f"decode after {which} overflow")
    finally:
        m.close()


def test_create_frees_everything_on_allocation_failure():
    import nvfp4_mixture_experts_03_b200 as nv
    import torch
    dims, layer = _layer()
    lg = layer.to(DEV)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    try:
        for n in (1, 2):   # the status block, then the decode state
            nv.nvfp4_moe_test_fail_alloc(n)
            with pytest.raises(nv.NVFP4MoEError) as e:
                nv.MoELayer.from_layer(lg, top_k=dims.K, max_tokens=8)
            assert e.value.code == CUDA_ERR
    finally:
        nv.nvfp4_moe_test_fail_alloc(0)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0 - (4 << 20)   # nothing large left behind
    m = nv.MoELayer.from_layer(lg, top_k=dims.K, max_tokens=8)
    m.close()
