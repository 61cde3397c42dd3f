"""The allocation-free decode entry point, nvfp4_moe_forward_decode_static.

It serves callers that cannot allocate device memory at all -- code embedded in
a runtime that owns every device allocation, or that runs where cudaMalloc is
not allowed -- so they can neither create a handle (creation allocates a small
status block and the decode state) nor hand the layer a workspace.

The main check runs in a fresh child process, so no earlier test (and no handle)
has touched the library on the device: the child makes two static calls in a row
on the 512-expert, hidden 2048, intermediate 768, top-10 layer (8 tokens, then
1 token; the second call reuses the static scratch, which still holds the first
call's contents) before any handle exists, then creates a regular handle and
requires both static outputs to match the regular entry point (handle + caller
workspace) and the FP64 oracle within the parity tolerance. It lives in a file
of its own that pytest collects last.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _child():
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch

    import nvfp4_mixture_experts_03_b200 as nv
    import oracle
    import synth
    from helpers import assert_close

    wl = synth.CONFIGS["decode"]
    d = wl.dims
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    layer = synth.make_layer(d, synth.workload_seed(wl, 5), device=dev)
    cd = nv.Dims(d.H, d.I, d.E, d.K, nv.DECODE_MAX_T)
    cw = nv.Weights(*[t.data_ptr() for t in layer.planes()])
    stream = torch.cuda.current_stream().cuda_stream
    calls = []
    for call, T in enumerate((8, 1)):
        seed = synth.workload_seed(wl, 5) + 100 + call
        x = synth.make_x_bf16(T, d.H, seed, outliers=True, device=dev)
        logits = synth.make_logits(T, d.E, seed, zipf_s=wl.zipf_s, device=dev)
        got = torch.full((T, d.H), float("nan"), dtype=torch.float32, device=dev)
        io = nv.IO(T, nv.ACT_BF16, x.data_ptr(), None, logits.data_ptr(), None, None,
                   nv.OUT_F32, got.data_ptr(), None, None, None, None, None)
        rc = nv.nvfp4_moe_forward_decode_static(cd, cw, io, stream)
        assert rc == 0, f"static call {call + 1}: {nv.nvfp4_moe_strerror(rc)}"
        calls.append((x, logits, got))
    torch.cuda.synchronize()
    # only now a regular handle: the static calls above ran without one
    regular = nv.MoELayer.from_layer(layer, top_k=d.K, max_tokens=nv.DECODE_MAX_T)
    lc = layer.to("cpu")
    for call, (x, logits, got) in enumerate(calls):
        want = regular.forward(x, logits=logits)
        assert regular.status() == 0
        g = got.double().cpu().numpy()
        assert_close(g, want.double().cpu().numpy(), f"static vs regular, call {call + 1}")
        ref = oracle.forward(lc, x.cpu(), K=d.K, logits=logits.cpu())["out"]
        l2, mr = assert_close(g, ref, f"static vs oracle, call {call + 1}")
        print(f"call {call + 1} (T={x.shape[0]}): vs oracle l2 {l2:.2e} maxrel {mr:.2e}")
    regular.close()
    print("CHILD_OK")


def test_static_decode_in_fresh_process_matches_regular_and_oracle():
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "--child"], cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    print(r.stdout[-2000:])
    assert r.returncode == 0 and "CHILD_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


def test_static_decode_rejects_layers_outside_the_decode_kernel():
    import torch

    import nvfp4_mixture_experts_03_b200 as nv
    fake = nv.Weights(*[(1 << 40) + i * (1 << 30) for i in range(9)])
    x = torch.zeros(1, dtype=torch.uint8, device="cuda")
    io = nv.IO(8, nv.ACT_BF16, x.data_ptr(), None, x.data_ptr(), None, None, nv.OUT_F32,
               x.data_ptr(), None, None, None, None, None)
    wide = nv.Dims(9216, 768, 64, 8, 8)           # its activation tile exceeds the kernel's shared memory
    assert nv.nvfp4_moe_forward_decode_static(wide, fake, io, 0) == -2
    small = nv.Dims(256, 128, 8, 2, 16)
    io.T = 9                                          # beyond the decode path
    assert nv.nvfp4_moe_forward_decode_static(small, fake, io, 0) == -2


if __name__ == "__main__" and "--child" in sys.argv:
    _child()
