"""Shared helpers for the parity tests: tolerance metrics and a runner that feeds
one seeded input draw to both the CUDA layer (through the C ABI) and the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

# Floating-point bar (normalised L2 and max elementwise relative error against the
# FP64 oracle). The relative error of an element is |g - o| / max(|o|, rms(o)):
# the raw ratio is unbounded where the exact output crosses zero.
TOL_L2 = 2e-3
TOL_MAXREL = 1e-2
# Routing weights: FP32 softmax of at most 16 terms against FP64.
TOL_W = 2e-6


def metrics(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    denom = np.maximum(np.abs(ref), rms)
    l2 = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    maxrel = float(np.max(np.abs(got - ref) / np.maximum(denom, 1e-300))) if ref.size else 0.0
    return float(l2), maxrel


def assert_close(got, ref, what=""):
    l2, mr = metrics(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert l2 <= TOL_L2 and mr <= TOL_MAXREL, f"{what}: l2={l2:.3e} maxrel={mr:.3e}"
    return l2, mr


def run_gpu(layer_gpu, x, *, K, logits=None, ids=None, wts=None, x_scale=None, max_tokens=None,
            out=None, accumulate=False, flags=0):
    """Runs the CUDA layer with debug routing outputs; returns (out, debug dict, status).
    `flags`: test flags of include/nvfp4_moe_test.h set on the handle first."""
    import nvfp4_mixture_experts_03_b200 as nv
    T = x.shape[0]
    E = layer_gpu.dims.E
    m = nv.MoELayer.from_layer(layer_gpu, top_k=K, max_tokens=max_tokens or max(T, 1))
    if flags:
        assert nv.nvfp4_moe_test_set_flags(m.handle, flags) == 0
    dbg = nv.debug_buffers(T, E, K, x.device)
    o = m.forward(x, logits=logits, topk_ids=ids, topk_weights=wts, x_scale=x_scale, out=out,
                  accumulate=accumulate, debug=dbg)
    st = m.status()
    torch.cuda.synchronize()
    res = o.double().cpu().numpy(), {k: v.cpu() for k, v in dbg.items()}, st
    m.close()
    return res


def check_routing(dbg, ref, T, K):
    assert np.array_equal(dbg["ids"].numpy(), ref["ids"]), "top-k ids differ"
    assert np.array_equal(dbg["counts"].numpy(), ref["counts"]), "counts differ"
    assert np.array_equal(dbg["offsets"].numpy(), ref["offsets"]), "offsets differ"
    assert np.array_equal(dbg["perm"].numpy(), ref["perm"]), "permutation differs"
    np.testing.assert_allclose(dbg["w"].numpy(), ref["w"], rtol=TOL_W, atol=1e-7)
