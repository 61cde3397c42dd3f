"""Fault paths on the GPU, driven by the test hooks of include/nvfp4_moe_test.h.
No test here faults, traps or hangs a GPU: the decode test makes a bounded wait
run out (about 200 ms) and checks that the call reports TIMEOUT and that the
handle is correct again afterwards; the allocation test makes create's device
allocations fail one at a time."""
import pytest

import oracle
import synth
from helpers import assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda"
TIMEOUT, CUDA_ERR = -8, -5


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
        assert nv.nvfp4_moe_test_set_flags(m.handle, 8) == -1   # unknown flag
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
