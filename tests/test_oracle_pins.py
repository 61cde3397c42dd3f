"""Pins for the FP64 oracle: each test checks it against something other than
itself -- the public format tables, library routines (torch dtypes, numpy sorts,
torch softmax), a dense brute-force formulation, closed forms and invariances.
Negative controls plant mistakes in the oracle and require a pin to catch them."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import brute
from conftest import golden


def _read_golden(name):
    rows = []
    for line in open(golden(name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        rows.append((int(a, 16), float(b)))
    return rows


# ----------------------------------------------------------------- formats

def test_e2m1_table_matches_ocp_mx():
    rows = _read_golden("e2m1_ocp_mx.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e4m3_all_bytes_vs_torch_float8():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.to(torch.float64).numpy()
    for b in range(256):
        got = oracle.e4m3(b)
        if np.isnan(ref[b]):
            assert math.isnan(got), b
        else:
            assert got == ref[b], (b, got, ref[b])


def test_e4m3_golden_points():
    for b, val in _read_golden("e4m3_ocp_fp8.txt"):
        got = oracle.e4m3(b)
        assert (math.isnan(got) and math.isnan(val)) or got == val, (hex(b), got, val)


def test_bf16_decode_vs_torch():
    g = torch.Generator().manual_seed(5)
    bits = torch.randint(0, 1 << 16, (4000,), generator=g, dtype=torch.int32)
    ref = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    for b, r in zip(bits.tolist(), ref):
        got = oracle.bf16(b)
        assert (math.isnan(got) and math.isnan(r)) or got == r


def test_bf16_rne_vs_torch():
    g = torch.Generator().manual_seed(6)
    f = torch.randn(20000, generator=g, dtype=torch.float32) * torch.exp2(
        torch.randint(-20, 20, (20000,), generator=g).to(torch.float32))
    # add exact halfway cases: bf16 value + half an ulp, both parities
    base = f[:2000].to(torch.bfloat16).to(torch.float32)
    ulp = torch.abs(base) * 2.0 ** -8
    f = torch.cat([f, base + torch.exp2(torch.floor(torch.log2(ulp)))])
    ref = f.to(torch.bfloat16).view(torch.int16).to(torch.int32).numpy() & 0xFFFF
    for v, r in zip(f.tolist(), ref):
        assert oracle.bf16_rne(v) == r, (v, oracle.bf16_rne(v), r)


def test_bf16_rne_array_matches_scalar():
    g = np.random.default_rng(7)
    v = g.standard_normal(5000) * np.exp2(g.integers(-30, 30, 5000))
    bits = oracle.bf16_rne_array(v)
    assert all(int(b) == oracle.bf16_rne(float(x)) for b, x in zip(bits[:500], v[:500]))
    # a value exactly halfway between two BF16 neighbours, in FP64 only (no FP32 detour)
    lo = 1.0 + 2.0 ** -7                # BF16 1.0078125 (odd last bit)
    assert oracle.bf16_rne_array(np.array([lo + 2.0 ** -8]))[0] == 0x3F82   # tie -> even (1.015625)
    assert oracle.bf16_rne_array(np.array([1.0 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81


def test_decode_matrix_equals_dense_library_decode():
    """The oracle's whole-matrix decoder against the brute-force decoder (numpy
    nibble split, OCP MX magnitude table, torch.float8_e4m3fn scales), element by
    element in FP64, on random planes that include a zero group, a negative-scale
    byte and a NaN scale byte (each must decode the same way on both sides)."""
    g = np.random.default_rng(8)
    rows, cols = 24, 96
    codes = g.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    scales = g.integers(0, 0x7F, (rows, cols // 16), dtype=np.uint8)
    codes[3, 8:16] = 0                 # a group of zero codes (group 1 of row 3)
    scales[5, 2] = 0                   # a zero scale
    scales[7, 1] = 0xB8                # -1.0: a sign bit set
    scales[9, 4] = 0x7F                # NaN
    for glob in (1.0, 3.0517578125e-05, -0.75):
        got = oracle.decode_matrix(codes, scales, glob)
        ref = brute.dense(codes, scales, glob)
        same = (got == ref) | (np.isnan(got) & np.isnan(ref))
        assert same.all(), (glob, np.argwhere(~same)[:4])
    assert np.all(oracle.decode_matrix(codes, scales, 1.0)[3, 16:32] == 0.0)


def test_dequant_products_exact_in_fp16_and_bf16():
    """code x scale has at most 6 significant bits and lies in [2^-10, 2688]: it is
    exact in both 16-bit float formats (checked exhaustively over 16 x 126 pairs)."""
    for c in range(16):
        for s in range(0x7F):
            v = oracle.e2m1(c) * oracle.e4m3(s)
            assert float(torch.tensor(v, dtype=torch.float64).to(torch.float16)) == v
            assert float(torch.tensor(v, dtype=torch.float64).to(torch.bfloat16)) == v


# --------------------------------------------------------------- quantiser

def _weights(seed, shape, std=0.02):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)


def test_generator_quantiser_equals_oracle_quantiser():
    w = _weights(1, (3, 40, 64))
    w[1, 3, :16] = 0                      # a zero group
    w[1, 4, 16:32] = 1e-30                # a group that underflows E4M3
    w[2] *= 1000.0                        # a different global
    c, s, gl = synth.quantize_nvfp4(w)
    oc, os_, og = oracle.quantize(w)
    assert np.array_equal(c.numpy(), oc)
    assert np.array_equal(s.numpy(), os_)
    assert np.array_equal(gl.numpy(), og)


def test_quantiser_round_trip_and_error_bound():
    w = _weights(2, (1, 32, 128))
    c, s, gl = oracle.quantize(w)
    W = brute.dense(c[0], s[0], gl[0])
    w64 = w[0].to(torch.float64).numpy()
    # error <= half the largest E2M1 gap (2, between 4 and 6) x scale x global,
    # and <= half the local gap for values inside the grid
    step = np.repeat(np.array([[oracle.e4m3(int(b)) for b in row] for row in s[0]]), 16, 1) * gl[0]
    assert np.all(np.abs(W - w64) <= 1.0 * step + 1e-30)
    # the global maximum maps to code +-6 exactly at scale 448
    r, k = np.unravel_index(np.argmax(np.abs(w64)), w64.shape)
    nib = (c[0, r, k // 2] >> (4 * (k & 1))) & 0xF
    assert oracle.e2m1(int(nib)) in (6.0, -6.0)
    assert s[0, r, k // 16] == 0x7E
    # re-quantising the decoded weights (as BF16) reproduces the codes and scales
    c2, s2, g2 = oracle.quantize(torch.from_numpy(W).to(torch.bfloat16)[None])
    assert np.array_equal(s2, s) and np.array_equal(g2, gl)
    lo = lambda a: np.stack([a & 0xF, a >> 4], -1)
    n1, n2 = lo(c), lo(c2)
    same = (n1 == n2) | ((n1 & 7) == 0) & ((n2 & 7) == 0)   # +0 / -0 are one value
    assert np.all(same)


# ------------------------------------------- activation formats (FP4 x FP4 study)

_E2M1_VALS = np.array([v for m in brute.E2M1_MAGNITUDES for v in (m, -m)])


def test_nvfp4_activations_exact_values_round_trip():
    # rows built from exact NVFP4 values: each block holds a +-6 code so that its
    # amax is 6 x its E4M3 scale x a power-of-two global, and one block per row
    # sits at scale 448 so that the global is amax / (6 * 448) exactly
    g = torch.Generator().manual_seed(11)
    T, H = 3, 64
    mags = torch.tensor(brute.E2M1_MAGNITUDES, dtype=torch.float64)
    e4 = torch.arange(1, 127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    e4 = e4.to(torch.float64)
    x = torch.zeros(T, H, dtype=torch.float64)
    for t in range(T):
        glob = 2.0 ** (-12 + 3 * t)
        for b in range(H // 16):
            sc = 448.0 if b == t % (H // 16) else float(e4[torch.randint(0, len(e4), (1,), generator=g)])
            v = mags[torch.randint(0, 8, (16,), generator=g)]
            v = v * torch.where(torch.rand(16, generator=g) < 0.5, -1.0, 1.0)
            v[int(torch.randint(0, 16, (1,), generator=g))] = 6.0
            x[t, 16 * b:16 * b + 16] = v * sc * glob
    xb = x.to(torch.bfloat16)
    assert torch.equal(xb.to(torch.float64), x)          # exact in BF16
    c, s, gl = oracle.quantize_act_nvfp4(xb)
    assert np.array_equal(oracle.dequant_act_nvfp4(c, s, gl), x.numpy())
    assert np.array_equal(gl.astype(np.float64), [2.0 ** (-12 + 3 * t) for t in range(T)])


def test_nvfp4_activations_pick_the_nearest_block_scale_and_code():
    x = synth.make_x_bf16(5, 128, seed=12, outliers=True)
    c, s, gl = oracle.quantize_act_nvfp4(x)
    xf = x.to(torch.float64).numpy()
    e4 = torch.arange(0, 127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    e4 = e4.to(torch.float64).numpy()
    for t in range(5):
        assert gl[t] == np.float32(np.abs(xf[t]).max() / (6.0 * 448.0))
        g = float(gl[t])
        for b in range(128 // 16):
            blk = xf[t, 16 * b:16 * b + 16]
            want = np.abs(blk).max() / g / 6.0
            sb = int(s[t, b])
            assert abs(e4[sb] - want) <= np.abs(e4 - want).min()   # nearest E4M3 scale
            step = e4[sb] * g
            q = brute.dense(c[t:t + 1, 8 * b:8 * b + 8], s[t:t + 1, b:b + 1], g)[0]
            for k in range(16):                                     # nearest code at that scale
                assert abs(q[k] - blk[k]) <= np.abs(_E2M1_VALS * step - blk[k]).min() * (1 + 1e-12)


def test_int8_activations_round_trip_and_half_step_bound():
    q0 = torch.randint(-127, 128, (4, 96), generator=torch.Generator().manual_seed(13))
    q0[:, 5] = 127
    sc = torch.tensor([2.0 ** -7, 2.0 ** -3, 0.5, 4.0], dtype=torch.float64)
    x = (q0.to(torch.float64) * sc[:, None]).to(torch.bfloat16)
    assert torch.equal(x.to(torch.float64), q0.to(torch.float64) * sc[:, None])
    q, s = oracle.quantize_act_int8(x)
    assert np.array_equal(q.astype(np.int64), q0.numpy()) and np.array_equal(s, sc.numpy())
    y = synth.make_x_bf16(6, 200, seed=14, outliers=True)
    q, s = oracle.quantize_act_int8(y)
    yf = y.to(torch.float64).numpy()
    err = np.abs(q.astype(np.float64) * s[:, None].astype(np.float64) - yf)
    assert np.all(err <= 0.5 * s[:, None].astype(np.float64) * (1 + 1e-6))
    assert np.all(np.abs(q).max(axis=1) == 127)


def test_fp8_h_equals_library_float8_rounding_incl_ties():
    rng = np.random.default_rng(15)
    h = rng.standard_normal((4, 96)) * np.array([[1e-3], [1.0], [30.0], [1e4]])
    c, s = oracle.quantize_h_e4m3_rows(h)
    r = h / s.astype(np.float64)[:, None]
    # exact midpoints between neighbouring E4M3 values, both signs: ties go to the even byte
    pos = np.array([oracle.e4m3(b) for b in range(127)])
    mids = (pos[1:] + pos[:-1]) / 2.0
    r2 = np.concatenate([r, np.stack([mids[:96], -mids[20:116]])])
    r2 = np.clip(r2, -448.0, 448.0)
    r2[:, 0] = 448.0                                  # keep every row's scale at 1
    c2, s2 = oracle.quantize_h_e4m3_rows(r2)
    assert np.all(s2 == 1.0)
    lib = lambda v: torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.dequant_h_e4m3_rows(c2, s2), lib(r2))
    assert np.array_equal(oracle.dequant_h_e4m3_rows(c, s), lib(r) * s.astype(np.float64)[:, None])


def test_int8_h_blocks_round_trip_bound_and_finite_fp16_scale():
    rng = np.random.default_rng(16)
    q0 = rng.integers(-127, 128, (3, 64))
    q0[:, 7] = 127
    q0[:, 40] = -127
    d0 = np.array([[2.0 ** -10, 3.0], [0.75, 2.0 ** -3], [96.0, 0.5]])   # exact in FP16, one per block
    h = (q0.reshape(3, 2, 32) * d0[:, :, None]).reshape(3, 64)
    q, d = oracle.quantize_h_int8_blocks(h)
    assert np.array_equal(q.astype(np.int64), q0) and np.array_equal(d.astype(np.float64), d0)
    y = rng.standard_normal((5, 96)) * rng.exponential(1.0, (5, 1))
    q, d = oracle.quantize_h_int8_blocks(y)
    err = np.abs(oracle.dequant_h_int8_blocks(q, d) - y).reshape(5, 3, 32)
    dd = d.astype(np.float64)
    amax = np.abs(y).reshape(5, 3, 32).max(axis=2)
    assert np.all(np.abs(dd - amax / 127.0) <= np.abs(amax / 127.0) * 2.0 ** -11)   # FP16 nearest
    # half a step, plus the clamp when rounding d down pushed amax / d past 127
    assert np.all(err <= (0.5 * dd + np.maximum(amax - 127.0 * dd, 0.0))[:, :, None] * (1 + 1e-12))
    big = np.full((1, 32), 1e12)
    big[0, 3] = -1e12
    q, d = oracle.quantize_h_int8_blocks(big)      # the scale stays finite, the codes saturate
    assert np.isfinite(d.astype(np.float64)).all() and d[0, 0] == np.float16(65504.0)
    assert np.all(np.abs(q) == 127) and q[0, 3] == -127
    q, d = oracle.quantize_h_int8_blocks(np.zeros((1, 32)))
    assert d[0, 0] == 0 and not q.any()
    q, s = oracle.quantize_h_int8_rows(h)
    assert np.all(np.abs(q).max(axis=1) == 127)
    assert np.all(np.abs(q * s.astype(np.float64)[:, None] - h) <= 0.5 * s.astype(np.float64)[:, None] * (1 + 1e-6))


def test_layer_with_h_unrounded_is_the_oracle_layer():
    d = synth.LayerDims(E=6, H=64, I=48, K=3)
    layer = synth.make_layer(d, seed=17)
    x = synth.make_x_bf16(5, 64, seed=18)
    ids, w = synth.make_topk(5, 6, 3, seed=19)
    ref = oracle.moe(layer, x, ids, w.double(), K=3)
    out, neg = oracle.layer_with_h(layer, x, ids, w, K=3, sample=range(5), h_rounds=(None, lambda h: -h))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_allclose(neg, -ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())   # linear in h


# ----------------------------------------------------------------- routing

def test_route_matches_library_sort_and_softmax():
    l = synth.make_logits(50, 33, seed=3, zipf_s=1.1)
    l[7, :] = 0.5                         # all ties
    l[9, 4] = l[9, 20] = 9.0              # a tie at the top
    ids, w, bad = oracle.route(l, 5)
    assert bad == 0
    G = brute.gate_matrix(l, 5)
    for t in range(50):
        order = np.lexsort((np.arange(33), -l[t].numpy().astype(np.float64)))[:5]
        assert list(ids[t]) == list(order)
        np.testing.assert_allclose(w[t], G[t, ids[t]], rtol=1e-14, atol=0)
    assert list(ids[7]) == [0, 1, 2, 3, 4]
    np.testing.assert_allclose(w[7], 0.2, rtol=1e-15)
    assert list(ids[9][:2]) == [4, 20]
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)


def test_route_k_equals_e_is_full_softmax():
    l = synth.make_logits(20, 12, seed=4)
    ids, w, _ = oracle.route(l, 12)
    full = torch.softmax(l.to(torch.float64), dim=1).numpy()
    for t in range(20):
        np.testing.assert_allclose(w[t], full[t, ids[t]], rtol=1e-13)
        assert sorted(ids[t]) == list(range(12))


def test_route_nonfinite_flagged():
    l = synth.make_logits(4, 8, seed=5)
    l[1, 3] = float("nan")
    l[2, 5] = float("inf")
    ids, w, bad = oracle.route(l, 2)
    assert 3 not in ids[1]          # NaN ranks below every number
    assert ids[2][0] == 5 and bad == 1


def test_sort_matches_stable_library_sort():
    ids, _ = synth.make_topk(300, 40, 6, seed=7)
    counts, offsets, perm = oracle.sort(ids, 40)
    flat = ids.numpy().reshape(-1)
    ref = np.argsort(flat, kind="stable")          # pair index t*K+j; stable keeps t order
    assert np.array_equal(perm, ref)
    assert counts.sum() == 300 * 6 and np.array_equal(np.bincount(flat, minlength=40), counts)
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(np.sort(perm), np.arange(300 * 6))
    assert np.all(np.bincount(perm // 6, minlength=300) == 6)   # every token K times
    assert np.all(np.diff(flat[perm]) >= 0)                     # grouped by expert ascending


def test_check_ids():
    ids, _ = synth.make_topk(10, 16, 4, seed=8)
    assert oracle.check_ids(ids, 16) == 0
    bad = ids.clone()
    bad[2, 1] = bad[2, 0]
    bad[5, 3] = 16
    assert oracle.check_ids(bad, 16) == 2


# ------------------------------------------------------------------- layer

def _tiny(seed=11, dims=synth.TINY):
    return synth.make_layer(dims, seed)


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("act", ["bf16", "int8"])
def test_layer_matches_dense_brute_force(act):
    layer = _tiny()
    T, K = 24, 2
    logits = synth.make_logits(T, 8, seed=12)
    if act == "bf16":
        x = synth.make_x_bf16(T, 256, seed=13)
        xs, X = None, brute.bf16_to_f64(x)
    else:
        x, xs = synth.make_x_int8(T, 256, seed=13)
        X = x.numpy().astype(np.float64) * xs.numpy().astype(np.float64)[:, None]
    r = oracle.forward(layer, x, K=K, logits=logits, x_scale=xs)
    ref = brute.layer_out(layer, X, brute.gate_matrix(logits, K))
    assert _rel(r["out"], ref) < 1e-12


def test_layer_precomputed_routing_and_sample():
    layer = _tiny()
    ids, w = synth.make_topk(16, 8, 3, seed=14)
    x = synth.make_x_bf16(16, 256, seed=15)
    full = oracle.moe(layer, x, ids, w, K=3)
    ref = brute.layer_out(layer, brute.bf16_to_f64(x), brute.gate_matrix_from(ids, w, 8))
    assert _rel(full, ref) < 1e-12
    part = oracle.moe(layer, x, ids, w, K=3, sample=[5, 0, 11])
    assert np.array_equal(part, full[[5, 0, 11]])


def test_single_expert_is_plain_swiglu_ffn():
    dims = synth.LayerDims(E=1, H=128, I=128, K=1)
    layer = synth.make_layer(dims, seed=16, keep_bf16=True)
    x = synth.make_x_bf16(9, 128, seed=17)
    ids = torch.zeros(9, 1, dtype=torch.int32)
    w = torch.ones(9, 1)
    out = oracle.moe(layer, x, ids, w, K=1)
    Wg = brute.dense(layer.gate_codes[0], layer.gate_scales[0], layer.gate_global[0])
    Wu = brute.dense(layer.up_codes[0], layer.up_scales[0], layer.up_global[0])
    Wd = brute.dense(layer.down_codes[0], layer.down_scales[0], layer.down_global[0])
    X = torch.from_numpy(brute.bf16_to_f64(x))
    h = torch.nn.functional.silu(X @ torch.from_numpy(Wg).T) * (X @ torch.from_numpy(Wu).T)
    ref = (h @ torch.from_numpy(Wd).T).numpy()
    assert _rel(out, ref) < 1e-12
    # and the decoded weights are the BF16 weights to within the quantiser's error
    assert _rel(Wg, layer.bf16["gate"][0].double().numpy()) < 0.2


def test_unit_scales_reduce_to_code_table():
    """All scales 1.0 (E4M3 0x38) and globals 1: G is the code table itself; with
    every code 2 (value 1.0) and x = 1, g = u = H and y = I * SiLU(H) * H."""
    E, H, I = 1, 128, 128
    mk = lambda shape, v: torch.full(shape, v, dtype=torch.uint8)
    layer = synth.Layer(synth.LayerDims(E, H, I, 1),
                        gate_codes=mk((E, I, H // 2), 0x22), up_codes=mk((E, I, H // 2), 0x22),
                        gate_scales=mk((E, I, H // 16), 0x38), up_scales=mk((E, I, H // 16), 0x38),
                        gate_global=torch.ones(E), up_global=torch.ones(E),
                        down_codes=mk((E, H, I // 2), 0x22), down_scales=mk((E, H, I // 16), 0x38),
                        down_global=torch.ones(E))
    x = torch.ones(2, H, dtype=torch.bfloat16)
    out = oracle.moe(layer, x, torch.zeros(2, 1, dtype=torch.int32), torch.ones(2, 1), K=1)
    silu_H = 128.0  # sigmoid(128) == 1.0 in FP64
    np.testing.assert_allclose(out, I * silu_H * 128.0, rtol=1e-15)


def test_expert_relabelling_invariance():
    layer = _tiny()
    logits = synth.make_logits(20, 8, seed=18)
    x = synth.make_x_bf16(20, 256, seed=19)
    base = oracle.forward(layer, x, K=2, logits=logits)["out"]
    p = torch.randperm(8, generator=torch.Generator().manual_seed(3))
    perm_layer = synth.Layer(layer.dims, **{k: getattr(layer, k)[p] for k in (
        "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global", "up_global",
        "down_codes", "down_scales", "down_global")})
    out = oracle.forward(perm_layer, x, K=2, logits=logits[:, p])["out"]
    assert _rel(out, base) < 1e-13


def test_token_permutation_equivariance():
    layer = _tiny()
    logits = synth.make_logits(20, 8, seed=20)
    x = synth.make_x_bf16(20, 256, seed=21)
    base = oracle.forward(layer, x, K=2, logits=logits)["out"]
    p = torch.randperm(20, generator=torch.Generator().manual_seed(4))
    out = oracle.forward(layer, x[p], K=2, logits=logits[p])["out"]
    assert np.array_equal(out, base[p.numpy()])


def test_global_power_of_two_scales_exactly():
    layer = _tiny()
    logits = synth.make_logits(10, 8, seed=22)
    x = synth.make_x_bf16(10, 256, seed=23)
    base = oracle.forward(layer, x, K=2, logits=logits)["out"]
    l2 = synth.Layer(layer.dims, **{k: getattr(layer, k) for k in (
        "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global", "up_global",
        "down_codes", "down_scales")}, down_global=layer.down_global * 8.0)
    out = oracle.forward(l2, x, K=2, logits=logits)["out"]
    assert np.array_equal(out, base * 8.0)


# -------------------------------------------------------- negative controls

@pytest.mark.parametrize("plant", ["nibble_order", "group_shift", "no_global", "swap_gate_up",
                                   "silu_sign", "equal_weights"])
def test_planted_mistake_is_caught_by_brute_force(plant):
    layer = _tiny()
    logits = synth.make_logits(16, 8, seed=24)
    x = synth.make_x_bf16(16, 256, seed=25)
    ref = brute.layer_out(layer, brute.bf16_to_f64(x), brute.gate_matrix(logits, 2))
    good = oracle.forward(layer, x, K=2, logits=logits)["out"]
    bad = oracle.forward(layer, x, K=2, logits=logits, plant=plant)["out"]
    assert _rel(good, ref) < 1e-12
    assert _rel(bad, ref) > 1e-2, plant


# ------------------------------------------------------------ router projection
# "Strata NVFP4" README, "How it differs from upstream Strata": the router's BF16
# projection takes FP32-exact inputs.

def _bf16_bits(a):
    return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_router_one_hot_rows_return_the_fp32_inputs_unrounded():
    """W_r row e is one-hot at column k_e (BF16 1.0): logit e of token t is x[t][k_e]
    itself. The inputs carry bits BF16 cannot hold, so rounding x to BF16 before the
    product (the mistake the pages' reading rules out) fails here."""
    H, E, T = 96, 7, 3
    rng = np.random.default_rng(5)
    x = rng.standard_normal((T, H)).astype(np.float32)
    x[:, ::5] = np.float32(1.0) + np.float32(2.0 ** -20)   # not representable in BF16
    w = np.zeros((E, H), np.uint16)
    cols = rng.choice(H, E, replace=False)
    cols[0] = 0                                             # one column hits the 1 + 2^-20 values
    w[np.arange(E), cols] = 0x3F80
    got = oracle.router(x, w)
    assert np.array_equal(got, x[:, cols].astype(np.float64))
    assert got[0, 0] == 1.0 + 2.0 ** -20


def test_router_all_ones_rows_are_exact_row_sums():
    """W_r of ones: every logit is the exactly rounded sum of the token's inputs."""
    H, E, T = 128, 3, 4
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((T, H)) * 3).astype(np.float32)
    w = np.full((E, H), 0x3F80, np.uint16)
    got = oracle.router(x, w)
    for t in range(T):
        want = math.fsum(float(v) for v in x[t])
        assert np.allclose(got[t], want, rtol=1e-13, atol=1e-12)


def test_router_matches_dense_fp64_product():
    """Random BF16 W_r [E][H] (E != H, so a transposed operand cannot pass) against
    a library FP64 matrix product of the decoded values."""
    T, E, H = 5, 24, 160
    rng = np.random.default_rng(7)
    x = rng.standard_normal((T, H)).astype(np.float32)
    wb = _bf16_bits(rng.standard_normal((E, H)) * 0.05)
    wf = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = x.astype(np.float64) @ wf.T
    got = oracle.router(x, wb)
    assert got.shape == (T, E)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-13)


def test_router_input_per_activation_type():
    """BF16 activations reach the router exactly; int8 codes as the FP32 product
    q * scale, one correctly rounded multiply."""
    rng = np.random.default_rng(8)
    xb = torch.from_numpy(rng.standard_normal((2, 64)).astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(oracle.router_input(xb), xb.float().numpy())
    q = torch.from_numpy(rng.integers(-127, 128, (2, 64)).astype(np.int8))
    s = torch.tensor([0.0123, 3.7], dtype=torch.float32)
    want = np.array([[float(np.float32(float(q[t, k]) * float(s[t]))) for k in range(64)]
                     for t in range(2)], np.float32)
    assert np.array_equal(oracle.router_input(q, s), want)


def test_router_logits_with_k_equal_e_route_to_the_full_softmax():
    """K = E: the routing weights of the router's logits are the softmax over all
    experts of those logits (rounded to FP32 for the selection)."""
    T, E, H = 3, 6, 64
    rng = np.random.default_rng(9)
    x = rng.standard_normal((T, H)).astype(np.float32)
    wb = _bf16_bits(rng.standard_normal((E, H)) * 0.1)
    l32 = oracle.router(x, wb).astype(np.float32).astype(np.float64)
    ids, w, bad = oracle.route(l32.astype(np.float32), E)
    assert bad == 0
    for t in range(T):
        sm = np.exp(l32[t] - l32[t].max())
        sm /= sm.sum()
        assert np.allclose(w[t], sm[ids[t]], rtol=1e-12, atol=1e-15)
        assert list(ids[t]) == sorted(range(E), key=lambda e: (-l32[t, e], e))
