"""A stack of decode layers in one kernel launch (nvfp4_moe_forward_decode_stack).

The stack kernel runs each layer's arithmetic exactly as the single-layer decode
kernel does, so its result must equal the layer-by-layer chain bit for bit: that
chain is built here from separate forward calls (out = y_l, then x_{l+1} = x_l + y_l
in FP32, the same add the layer performs in place), and each y_l is checked
against the FP64 oracle run on that layer's own input bf16(x_l).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _chain(models, x0, logits, layers_cpu=None, check=()):
    """Layer-by-layer forward calls; returns the final x and checks the listed
    layers' increments against the oracle."""
    x = x0.clone()
    for l, m in enumerate(models):
        y = m.forward(x, logits=logits[l])
        assert m.status() == 0
        if l in check:
            xb = x.to(torch.bfloat16).cpu()
            ref = oracle.forward(layers_cpu[l], xb, K=m.K, logits=logits[l].cpu())["out"]
            assert_close(y.double().cpu().numpy(), ref, f"layer {l}")
        x = x + y
    return x


@pytest.mark.parametrize("T", [1, 3, 8])
def test_stack_equals_layer_by_layer_and_oracle(T):
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.LayerDims(E=48, H=256, I=160, K=4)
    L = 5
    layers = [synth.make_layer(dims, seed=300 + l) for l in range(L)]
    models = [nv.MoELayer.from_layer(Ly.to(DEV), top_k=dims.K, max_tokens=8) for Ly in layers]
    x0 = synth.make_x_f32(T, dims.H, 310 + T, outliers=True).to(DEV)
    logits = torch.stack([synth.make_logits(T, dims.E, 320 + l) for l in range(L)]).to(DEV).contiguous()
    want = _chain(models, x0, logits, layers, check=range(L))
    x = x0.clone()
    nv.decode_stack(models, x, logits)
    assert models[0].status() == 0
    for m in models:
        m.close()
    assert torch.equal(x.view(torch.int32), want.view(torch.int32))


def test_stack_48_full_size_layers():
    """The benchmark stack: 48 layers of the 512-expert, hidden 2048, intermediate
    768, top-10 shape (about 61 GB of planes), two tokens."""
    import nvfp4_mixture_experts_03_b200 as nv
    wl = synth.CONFIGS["stack48"]
    d = wl.dims
    T = 2
    seed0 = synth.workload_seed(wl)
    layers = [synth.make_layer(d, synth.workload_seed(wl, l), device=DEV) for l in range(wl.layers)]
    models = [nv.MoELayer.from_layer(Ly, top_k=d.K, max_tokens=8) for Ly in layers]
    x0 = synth.make_x_f32(T, d.H, seed0 + 5, outliers=False, device=DEV).contiguous()
    logits = torch.stack([synth.make_logits(T, d.E, synth.workload_seed(wl, l) + 303, zipf_s=wl.zipf_s,
                                            device=DEV) for l in range(wl.layers)]).contiguous()
    check = (0, wl.layers - 1)
    cpu = {l: layers[l].to("cpu") for l in check}
    want = _chain(models, x0, logits, cpu, check=check)
    x = x0.clone()
    nv.decode_stack(models, x, logits)
    assert models[0].status() == 0
    assert bool(torch.isfinite(x).all())
    assert torch.equal(x.view(torch.int32), want.view(torch.int32))
    for m in models:
        m.close()


def test_stack_rejects_bad_calls():
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.LayerDims(E=16, H=256, I=128, K=2)
    a = nv.MoELayer.from_layer(synth.make_layer(dims, seed=330).to(DEV), top_k=2, max_tokens=8)
    b = nv.MoELayer.from_layer(synth.make_layer(synth.LayerDims(E=16, H=256, I=160, K=2), seed=331).to(DEV),
                               top_k=2, max_tokens=8)
    x = synth.make_x_f32(2, dims.H, 332, outliers=False).to(DEV)
    lg = torch.stack([synth.make_logits(2, dims.E, 333 + l) for l in range(2)]).to(DEV).contiguous()
    with pytest.raises(nv.NVFP4MoEError) as e:
        nv.decode_stack([a, b], x, lg)          # dims differ
    assert e.value.code == -1
    with pytest.raises(nv.NVFP4MoEError):
        nv.decode_stack([a, a], x.to(torch.bfloat16), lg)   # not the FP32 residual stream
    nv.decode_stack([a, a], x, lg)
    assert a.status() == 0
    a.close()
    b.close()
