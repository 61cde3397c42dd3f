"""Router projection on the GPU against the FP64 oracle.

The layer can compute its own router logits, logits[t][e] = sum_k W_r[e][k] x[t][k]
with W_r BF16 and x the layer's input in FP32, never rounded to BF16 ("Strata
NVFP4" README, "How it differs from upstream Strata"). The GPU accumulates in
FP32, so each logit is checked against the oracle's exact FP64 value within the
recursive-summation bound (H + 4) * 2^-24 * sum_k |W_r[e][k] x[t][k]| -- sixteen
times tighter, at H = 2048, than the error of rounding x to BF16 first.

Selection compares FP32 logits. A token whose K-th and (K+1)-th oracle logits lie
within twice that bound of each other may legitimately pick either, so ids are
required bit-exact (set and order) for every token whose top-(K+1) oracle logits
are separated by more than twice the bound; the other tokens' picks must each lie
within the bound of the K-th largest, and such tokens are left out of the output
comparison.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _x(kind, T, H, seed):
    if kind == "bf16":
        return synth.make_x_bf16(T, H, seed, outliers=True), None
    if kind == "f32":
        return synth.make_x_f32(T, H, seed, outliers=True), None
    return synth.make_x_int8(T, H, seed, outliers=True)


def _bound(x_f32, wr):
    w = wr.float().double().numpy()
    return (x_f32.shape[1] + 4) * 2.0 ** -24 * (np.abs(x_f32.astype(np.float64)) @ np.abs(w).T)


def _check_ids(ids_gpu, l64, bound, K):
    """-> mask of tokens whose selected set is unambiguous (checked bit-exact there:
    the set, and the order of every pair of selected logits further apart than
    twice the bound)."""
    T = l64.shape[0]
    clear = np.zeros(T, bool)
    for t in range(T):
        order = sorted(range(l64.shape[1]), key=lambda e: (-np.float32(l64[t, e]), e))
        b = 2 * bound[t].max()
        kth = l64[t, order[K - 1]]
        got = list(ids_gpu[t])
        assert len(set(got)) == K
        if kth - l64[t, order[K]] > b:
            clear[t] = True
            assert set(got) == set(order[:K]), f"token {t}: {got} vs {order[:K]}"
            for i in range(K):
                for j in range(i + 1, K):
                    if l64[t, got[i]] < l64[t, got[j]] - b:
                        raise AssertionError(f"token {t}: order {got} vs {order[:K]}")
        else:
            assert all(l64[t, e] >= kth - b for e in got), f"token {t}"
    return clear


@pytest.mark.parametrize("kind", ["bf16", "f32", "int8"])
@pytest.mark.parametrize("T", [1, 5, 8, 300])
def test_router_layer_matches_oracle(kind, T):
    """Small layer: logits, ids, weights and the layer output with the router
    projection computed by the library (T <= 8 takes the decode kernel, 300 the
    grouped GEMMs; 300 tokens span three 128-token GEMM tiles and a ragged one)."""
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.LayerDims(E=64, H=512, I=256, K=6)
    layer = synth.make_layer(dims, seed=90)
    x, xs = _x(kind, T, dims.H, seed=91 + T)
    wr = synth.make_router_w(dims.E, dims.H, seed=92)
    ref = oracle.forward(layer, x, K=dims.K, x_scale=xs, router_w=wr)
    m = nv.MoELayer.from_layer(layer.to(DEV), top_k=dims.K, max_tokens=max(T, 8))
    dbg = nv.debug_buffers(T, dims.E, dims.K, DEV)
    out = m.forward(x.to(DEV), x_scale=None if xs is None else xs.to(DEV), router_w=wr.to(DEV),
                    debug=dbg)
    assert m.status() == 0
    m.close()
    lg = dbg["logits"].double().cpu().numpy()
    bound = _bound(oracle.router_input(x, xs), wr)
    err = np.abs(lg - ref["logits64"])
    assert np.all(err <= bound + 1e-30), f"max err/bound {np.max(err / (bound + 1e-30)):.3f}"
    clear = _check_ids(dbg["ids"].cpu().numpy(), ref["logits64"], bound, dims.K)
    w = dbg["w"].double().cpu().numpy()
    assert np.allclose(w[clear], ref["w"][clear], rtol=1e-5, atol=1e-6)
    assert clear.sum() >= max(1, (3 * T) // 5)
    o = out.double().cpu().numpy()
    assert_close(o[clear], ref["out"][clear], f"router layer {kind} T={T}")


@pytest.mark.parametrize("T", [8, 8192])
def test_router_full_size_logits(T):
    """The benchmark layer's shape (512 experts, hidden 2048): the FP32 logits of
    sampled tokens (every 128-token tile's first and last token, plus the ragged
    end) against the oracle, and the selection of every sampled token."""
    import nvfp4_mixture_experts_03_b200 as nv
    wl = synth.CONFIGS["decode"]
    d = wl.dims
    x = synth.make_x_bf16(T, d.H, 93, outliers=True)
    wr = synth.make_router_w(d.E, d.H, seed=94)
    layer = synth.make_layer(synth.LayerDims(E=d.E, H=d.H, I=64, K=d.K), seed=95)
    m = nv.MoELayer.from_layer(layer.to(DEV), top_k=d.K, max_tokens=T)
    dbg = nv.debug_buffers(T, d.E, d.K, DEV)
    m.forward(x.to(DEV), router_w=wr.to(DEV), debug=dbg)
    assert m.status() == 0
    m.close()
    toks = sorted(set([t for t0 in range(0, T, 128) for t in (t0, min(t0 + 127, T - 1))] + [T - 1]))
    xf = oracle.router_input(x)[toks]
    l64 = oracle.router(xf, wr)
    bound = _bound(xf, wr)
    lg = dbg["logits"].double().cpu().numpy()[toks]
    assert np.all(np.abs(lg - l64) <= bound + 1e-30)
    clear = _check_ids(dbg["ids"].cpu().numpy()[toks], l64, bound, d.K)
    print(f"T={T}: {len(toks)} tokens checked, {int(clear.sum())} with an unambiguous selection")


def test_router_rejects_ambiguous_routing_sources():
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.LayerDims(E=16, H=256, I=128, K=2)
    layer = synth.make_layer(dims, seed=96)
    m = nv.MoELayer.from_layer(layer.to(DEV), top_k=dims.K, max_tokens=8)
    x = synth.make_x_bf16(2, dims.H, 97).to(DEV)
    wr = synth.make_router_w(dims.E, dims.H, seed=98).to(DEV)
    lg = synth.make_logits(2, dims.E, 99).to(DEV)
    with pytest.raises(nv.NVFP4MoEError) as e:
        m.forward(x, logits=lg, router_w=wr)
    assert e.value.code == -1
    ids, w = synth.make_topk(2, dims.E, dims.K, 100)
    with pytest.raises(nv.NVFP4MoEError):
        m.forward(x, topk_ids=ids.to(DEV), topk_weights=w.to(DEV), router_w=wr)
    m.close()
