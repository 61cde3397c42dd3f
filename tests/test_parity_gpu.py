"""GPU parity: the CUDA layer, called through the C ABI, against the FP64 oracle
on the same seeded inputs. Routing ids, counts, offsets and the permutation must
match bit for bit; routing weights to FP32 rounding; the layer output within
normalised L2 <= 2e-3 and max elementwise relative error <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close, check_routing, run_gpu

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(dims, T, seed, *, zipf=None, act="bf16", outliers=False):
    layer = synth.make_layer(dims, seed)
    logits = synth.make_logits(T, dims.E, seed, zipf_s=zipf)
    if act == "int8":
        x, xs = synth.make_x_int8(T, dims.H, seed, outliers=outliers)
    else:
        x, xs = synth.make_x_bf16(T, dims.H, seed, outliers=outliers), None
    return layer, logits, x, xs


NO_SMALL = 2   # include/nvfp4_moe_test.h: NVFP4_MOE_TEST_NO_SMALL


def _run_both(layer, logits, x, xs, K, **kw):
    ref = oracle.forward(layer, x, K=K, logits=logits, x_scale=xs)
    lg = layer.to(DEV)
    out, dbg, st = run_gpu(lg, x.to(DEV), K=K, logits=logits.to(DEV),
                           x_scale=None if xs is None else xs.to(DEV), **kw)
    return ref, out, dbg, st


# T <= 8 takes the decode (GEMV) path, larger T the grouped-GEMM path.
@pytest.mark.parametrize("T", [1, 3, 8, 9, 64, 200])
def test_tiny_layer_bf16(T):
    dims = synth.TINY
    layer, logits, x, xs = _case(dims, T, seed=synth.BASE_SEED + T)
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K)
    assert st == 0
    check_routing(dbg, ref, T, dims.K)
    assert_close(out, ref["out"], f"tiny T={T}")


@pytest.mark.parametrize("T", [2, 64])
def test_tiny_layer_int8(T):
    dims = synth.TINY
    layer, logits, x, xs = _case(dims, T, seed=700 + T, act="int8", outliers=True)
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K)
    assert st == 0
    check_routing(dbg, ref, T, dims.K)
    assert_close(out, ref["out"], f"tiny int8 T={T}")


@pytest.mark.parametrize("T", [5, 300])
def test_precomputed_routing(T):
    dims = synth.LayerDims(E=16, H=256, I=256, K=4)
    layer = synth.make_layer(dims, seed=31)
    x = synth.make_x_bf16(T, dims.H, seed=32)
    ids, w = synth.make_topk(T, dims.E, dims.K, seed=33)
    ref = oracle.forward(layer, x, K=dims.K, ids=ids, wts=w)
    out, dbg, st = run_gpu(layer.to(DEV), x.to(DEV), K=dims.K, ids=ids.to(DEV), wts=w.to(DEV))
    assert st == 0
    assert np.array_equal(dbg["perm"].numpy(), ref["perm"])
    assert np.array_equal(dbg["counts"].numpy(), ref["counts"])
    assert_close(out, ref["out"], "precomputed routing")


@pytest.mark.parametrize("T", [4, 700])
def test_medium_skewed_multi_tile(T):
    """Zipf-skewed routing: a hot expert spans several 256-pair tiles, a ragged
    last tile, and several experts stay empty."""
    dims = synth.LayerDims(E=64, H=512, I=384, K=6)
    layer, logits, x, xs = _case(dims, T, seed=41, zipf=1.1, outliers=True)
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K)
    assert st == 0
    check_routing(dbg, ref, T, dims.K)
    if T > 8:
        assert ref["counts"].max() > 256 and (ref["counts"] == 0).any()
    assert_close(out, ref["out"], f"medium T={T}")


@pytest.mark.parametrize("T", [3, 260])
def test_hidden_not_multiple_of_256(T):
    """H = 384: the down projection's last 256-row tile is half past H (its second
    CTA computes nothing that is kept); I = 128 is a single gate/up tile."""
    dims = synth.LayerDims(E=12, H=384, I=128, K=3)
    layer, logits, x, xs = _case(dims, T, seed=57, zipf=0.8)
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K)
    assert st == 0
    check_routing(dbg, ref, T, dims.K)
    assert_close(out, ref["out"], f"H=384 T={T}")


def test_one_expert_takes_every_token_and_k_equals_e():
    dims = synth.LayerDims(E=8, H=256, I=128, K=8)
    T = 40
    layer, logits, x, xs = _case(dims, T, seed=51)
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K)
    assert st == 0 and (ref["counts"] == T).all()
    check_routing(dbg, ref, T, dims.K)
    assert_close(out, ref["out"], "K = E")


def test_k1_single_hot_expert():
    dims = synth.LayerDims(E=8, H=256, I=128, K=1)
    T = 270
    layer, logits, x, xs = _case(dims, T, seed=52)
    logits[:, 5] += 100.0
    ref, out, dbg, st = _run_both(layer, logits, x, xs, 1)
    assert st == 0 and ref["counts"][5] == T
    check_routing(dbg, ref, T, 1)
    assert_close(out, ref["out"], "K = 1, one expert")


def test_residual_stream_accumulate():
    """x <- x + layer(bf16(x)) in place (act == out, FP32 residual)."""
    dims = synth.TINY
    T = 48
    layer, logits, _, _ = _case(dims, T, seed=53)
    x32 = synth.make_x_f32(T, dims.H, seed=54, outliers=False)
    xb = x32.to(torch.bfloat16)
    ref = oracle.forward(layer, xb, K=dims.K, logits=logits)
    xg = x32.to(DEV).contiguous()
    out, dbg, st = run_gpu(layer.to(DEV), xg, K=dims.K, logits=logits.to(DEV), out=xg,
                           accumulate=True)
    assert st == 0
    assert_close(out - x32.double().numpy(), ref["out"], "residual step")


def test_nonfinite_logit_is_reported():
    dims = synth.TINY
    T = 16
    layer, logits, x, _ = _case(dims, T, seed=55)
    logits[3, :] = float("nan")
    _, _, st = run_gpu(layer.to(DEV), x.to(DEV), K=dims.K, logits=logits.to(DEV))
    assert st == -7


def test_bad_precomputed_ids_are_reported_and_contained():
    dims = synth.TINY
    T = 12
    layer = synth.make_layer(dims, seed=56)
    x = synth.make_x_bf16(T, dims.H, seed=57)
    ids, w = synth.make_topk(T, dims.E, dims.K, seed=58)
    ids[2, 0] = 99
    ids[4, 1] = ids[4, 0]
    out, _, st = run_gpu(layer.to(DEV), x.to(DEV), K=dims.K, ids=ids.to(DEV), wts=w.to(DEV))
    assert st == -6
    assert np.all(out[[2, 4]] == 0.0) and np.all(np.isfinite(out))


def test_empty_batch_is_a_noop():
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.TINY
    layer = synth.make_layer(dims, seed=59).to(DEV)
    m = nv.MoELayer.from_layer(layer, top_k=dims.K, max_tokens=16)
    x = torch.empty(0, dims.H, dtype=torch.bfloat16, device=DEV)
    out = m.forward(x, logits=torch.empty(0, dims.E, device=DEV))
    assert out.shape == (0, dims.H) and m.status() == 0
    m.close()


def test_host_checks_on_device():
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.TINY
    layer = synth.make_layer(dims, seed=60).to(DEV)
    m = nv.MoELayer.from_layer(layer, top_k=dims.K, max_tokens=16)
    x = torch.zeros(17, dims.H, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(nv.NVFP4MoEError) as e:
        m.forward(x, logits=torch.zeros(17, dims.E, device=DEV))
    assert e.value.code == -1           # T > max_tokens
    x = torch.zeros(4, dims.H, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(nv.NVFP4MoEError) as e:
        m.forward(x, logits=torch.zeros(4, dims.E, device=DEV), workspace=ws)
    assert e.value.code == -4
    m.close()


def _scaled(layer, **factors):
    kw = {k: getattr(layer, k) for k in (
        "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global", "up_global",
        "down_codes", "down_scales", "down_global")}
    for k, f in factors.items():
        kw[k] = kw[k] * f
    return synth.Layer(layer.dims, **kw)


@pytest.mark.parametrize("T", [4, 12, 64])
@pytest.mark.parametrize("which", ["down", "gate_up"])
def test_f16_range_overflow_is_reported_never_silent(T, which):
    """Globals scaled by powers of two push the F16 intermediates past 65504: the
    down global pushes the grouped-GEMM path's per-pair rows w*s_d*y out of range
    (decode keeps y in FP32), the gate and up globals push h out of range on both
    paths. The result must be either correct (FP32 math kept it in range) or
    flagged NVFP4_MOE_ERR_NONFINITE -- never a silent inf in the output. T = 12
    leaves every expert with at most 16 pairs (the small-expert kernels), T = 64
    sends most of them through the tensor-core tiles."""
    dims = synth.TINY
    base, logits, x, _ = _case(dims, T, seed=63)
    if which == "down":
        layer = _scaled(base, down_global=2.0 ** 24)
    else:
        layer = _scaled(base, gate_global=2.0 ** 10, up_global=2.0 ** 10)
    ref = oracle.forward(layer, x, K=dims.K, logits=logits)
    out, dbg, st = run_gpu(layer.to(DEV), x.to(DEV), K=dims.K, logits=logits.to(DEV))
    assert np.abs(ref["out"]).max() > 65504.0 or which == "gate_up"
    if st == 0:
        assert_close(out, ref["out"], f"{which} scaled, T={T}")
    else:
        assert st == -7, st
    if not np.all(np.isfinite(out)):
        assert st == -7, "non-finite output without a NONFINITE status"
    if which == "gate_up":
        assert st == -7                 # h itself overflows F16 on both paths
    elif T > 8:
        assert st == -7                 # the per-pair F16 rows overflow


@pytest.mark.parametrize("T", [3, 8, 300])
def test_outputs_are_bitwise_reproducible(T):
    """Both paths add each token's expert rows in a fixed order with no
    floating-point atomics: the same call twice gives the same bits."""
    import nvfp4_mixture_experts_03_b200 as nv
    dims = synth.LayerDims(E=64, H=512, I=384, K=6)
    layer, logits, x, _ = _case(dims, T, seed=71, zipf=1.1, outliers=True)
    m = nv.MoELayer.from_layer(layer.to(DEV), top_k=dims.K, max_tokens=max(T, 8))
    xd, ld = x.to(DEV), logits.to(DEV)
    a = m.forward(xd, logits=ld).clone()
    b = m.forward(xd, logits=ld).clone()
    assert m.status() == 0
    m.close()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("T,flags", [(5, 0), (70, 0), (70, NO_SMALL), (20, 0)])
@pytest.mark.parametrize("H,I", [(160, 96), (224, 160), (256, 96), (160, 256), (96, 288)])
def test_hidden_and_inter_multiples_of_32(H, I, T, flags):
    """H and I that are multiples of 32 but not of 128: K rounds and K steps with a
    zero-padded tail, partial gate/up and down row tiles, and scale rows that are
    not 8-byte aligned. The last expert is made popular so the partial tiles at
    the very end of each plane are reached."""
    dims = synth.LayerDims(E=6, H=H, I=I, K=2)
    layer, logits, x, xs = _case(dims, T, seed=81 + H + I)
    logits[:, dims.E - 1] += 1.5
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K, flags=flags)
    assert st == 0
    assert ref["counts"][dims.E - 1] > 0
    check_routing(dbg, ref, T, dims.K)
    assert_close(out, ref["out"], f"H={H} I={I} T={T} flags={flags}")


@pytest.mark.parametrize("flags", [0, NO_SMALL])
@pytest.mark.parametrize("T", [24, 90, 700])
def test_small_experts_and_tiles(T, flags):
    """64 experts: at T = 24 (uniform routing) every expert has at most 16 pairs
    (all take the small-expert kernels); with Zipf-skewed routing at T = 90 the
    hot experts take the tensor-core tiles and the tail the small-expert kernels,
    at T = 700 most take the tiles. With NVFP4_MOE_TEST_NO_SMALL every expert
    takes the tiles. Every combination against the oracle."""
    dims = synth.LayerDims(E=64, H=512, I=384, K=6)
    layer, logits, x, xs = _case(dims, T, seed=91 + T, zipf=None if T == 24 else 1.1, outliers=True)
    ref, out, dbg, st = _run_both(layer, logits, x, xs, dims.K, flags=flags)
    assert st == 0
    check_routing(dbg, ref, T, dims.K)
    c = ref["counts"]
    small = int(((c > 0) & (c <= 16)).sum())
    if T == 24:
        assert c.max() <= 16
    else:
        assert small > 0 and c.max() > 16
    assert_close(out, ref["out"], f"small/tiles T={T} flags={flags}")
