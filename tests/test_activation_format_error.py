"""How far the layer moves when its activations are quantised the way a
block-scaled FP4 x FP4 prompt path (tcgen05 `kind::mxf4nvf4`) or the W4A8 path
needs them -- the accuracy half of the choice between block-scaled MMA and exact
dequantisation ("Strata NVFP4" README, "How it differs from upstream Strata", the
W4A8 bullet: 8-bit activations err far less per product than FP4 ones) -- and
when h, between the projections, is stored in 8 bits instead of F16 (the pages'
fused SwiGLU quantiser, "Strata NVFP4" README, the 0.1.39-nvfp4.2 bullet).

Each variant is evaluated exactly (FP64, dense brute-force formulation of the
layer) on activations rounded to its format, against the same layer on the BF16
activations themselves, so the figures are the formats' own error floor, before
any accumulation error of a kernel. Layer: the benchmark expert shape (H 2048,
I 768, top-10) with 16 experts; 24 tokens, with and without the 0.1 % outlier
channels of the synthetic workloads."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import brute

TOL_L2 = 2e-3   # the layer's parity tolerance (normalised L2)


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.fixture(scope="module")
def layer():
    return synth.make_layer(synth.LayerDims(E=16, H=2048, I=768, K=10), seed=21)


@pytest.mark.parametrize("outliers", [False, True])
def test_fp4_activations_miss_the_tolerance_int8_stays_closer(layer, outliers, capsys):
    T, E, K = 24, 16, 10
    x = synth.make_x_bf16(T, 2048, seed=22 + outliers, outliers=outliers)
    ids, w = synth.make_topk(T, E, K, seed=24)
    G = brute.gate_matrix_from(ids, w, E)
    x64 = brute.bf16_to_f64(x)
    c, s, g = oracle.quantize_act_nvfp4(x)
    x_fp4 = oracle.dequant_act_nvfp4(c, s, g)
    q, qs = oracle.quantize_act_int8(x)
    x_i8 = q.astype(np.float64) * qs.astype(np.float64)[:, None]
    out = brute.layer_out(layer, np.concatenate([x64, x_fp4, x_i8]), np.concatenate([G, G, G]))
    ref, o_fp4, o_i8 = out[:T], out[T:2 * T], out[2 * T:]
    e_fp4, e_i8 = _rel_l2(o_fp4, ref), _rel_l2(o_i8, ref)
    with capsys.disabled():
        print(f"\n[activation formats, outliers={outliers}] input rel L2: FP4 {_rel_l2(x_fp4, x64):.4f}"
              f" int8 {_rel_l2(x_i8, x64):.4f}; layer output rel L2: FP4 {e_fp4:.4f} int8 {e_i8:.4f}"
              f" (tolerance {TOL_L2})")
    assert e_fp4 > 10 * TOL_L2          # a block-scaled FP4 x FP4 path cannot meet the tolerance
    # 8-bit activations stay closer; with outlier channels a per-token int8 scale
    # spends most of its range on them and keeps less of that advantage
    assert e_i8 < (e_fp4 if outliers else e_fp4 / 5)


def test_eight_bit_h_needs_a_looser_tolerance_f16_h_does_not(layer, capsys):
    T, E, K = 8, 16, 10
    x = synth.make_x_bf16(T, 2048, seed=31)
    ids, w = synth.make_topk(T, E, K, seed=33)

    def rows_int8(h):
        q, s = oracle.quantize_h_int8_rows(h)
        return q.astype(np.float64) * s.astype(np.float64)[:, None]

    fmts = {
        "F16": lambda h: h.astype(np.float16).astype(np.float64),
        "int8, 32-blocks, FP16 scale": lambda h: oracle.dequant_h_int8_blocks(*oracle.quantize_h_int8_blocks(h)),
        "int8, per row": rows_int8,
        "E4M3, per row": lambda h: oracle.dequant_h_e4m3_rows(*oracle.quantize_h_e4m3_rows(h)),
    }
    outs = oracle.layer_with_h(layer, x, ids, w, K=K, sample=range(T), h_rounds=(None, *fmts.values()))
    ref = outs[0]
    err = {name: _rel_l2(o, ref) for name, o in zip(fmts, outs[1:])}
    with capsys.disabled():
        print("\n[h formats] layer output rel L2: " + ", ".join(f"{k} {v:.5f}" for k, v in err.items()))
    assert err["F16"] < TOL_L2 / 5                       # the product's F16 h leaves room
    assert TOL_L2 < err["int8, 32-blocks, FP16 scale"] < 5 * TOL_L2   # 8-bit h: a 1e-2 bound, not 2e-3
    assert err["int8, 32-blocks, FP16 scale"] < err["int8, per row"] < err["E4M3, per row"]


@pytest.mark.parametrize("outliers", [False, True])
def test_eight_bit_blocks_err_about_sixteen_times_less_than_fp4(outliers, capsys):
    # The pages put the W4A8 path's 8-bit activations at 16x smaller error per
    # product than FP4 ones ("Strata NVFP4" README, "How it differs from upstream
    # Strata", the W4A8 bullet). The 8-bit format read as llama.cpp's: blocks of
    # 32 with an FP16 scale; FP4 as per-token NVFP4. A product's error from its
    # activation is that activation's rounding error, so the ratio of the two
    # formats' element errors is the figure to compare.
    x = synth.make_x_bf16(24, 2048, seed=22 + outliers, outliers=outliers)
    x64 = brute.bf16_to_f64(x)
    x8 = oracle.dequant_h_int8_blocks(*oracle.quantize_h_int8_blocks(x64))
    x4 = oracle.dequant_act_nvfp4(*oracle.quantize_act_nvfp4(x))
    ratio = _rel_l2(x4, x64) / _rel_l2(x8, x64)
    with capsys.disabled():
        print(f"\n[8-bit vs FP4 activations, outliers={outliers}] element error ratio {ratio:.1f}")
    assert 8.0 < ratio < 32.0


def test_single_expert_with_eight_bit_blocks_brackets_the_pages_parity_error(capsys):
    # The pages report a three-expert CUDA parity of 1.096 %, 1.156 % and 1.159 %
    # relative output error against a 3 % threshold ("#2727 tools: add opt-in
    # FP4-Local CSF checkpoint conversion", "Validation") without saying what the
    # reference is. One plausible reading: their prompt path's 8-bit activations
    # (32-blocks, FP16 scales) against a float reference. One expert of the
    # benchmark shape, exact otherwise, with and without outlier channels:
    layer = synth.make_layer(synth.LayerDims(E=3, H=2048, I=768, K=1), seed=41)
    errs = {}
    for outliers in (False, True):
        x = synth.make_x_bf16(32, 2048, seed=42 + outliers, outliers=outliers)
        x64 = brute.bf16_to_f64(x)
        x8 = oracle.dequant_h_int8_blocks(*oracle.quantize_h_int8_blocks(x64))
        for e in range(3):
            G = np.zeros((32, 3))
            G[:, e] = 1.0
            o = brute.layer_out(layer, np.concatenate([x64, x8]), np.concatenate([G, G]))
            errs[(outliers, e)] = _rel_l2(o[32:], o[:32])
    with capsys.disabled():
        print("\n[one expert, 8-bit block activations] rel L2: " +
              ", ".join(f"{'outliers' if k[0] else 'plain'} e{k[1]} {100 * v:.2f} %" for k, v in errs.items()))
    plain = [v for k, v in errs.items() if not k[0]]
    outl = [v for k, v in errs.items() if k[0]]
    assert max(plain) < 0.011 < min(outl) and max(outl) < 0.03   # brackets 1.1 %, under the 3 % threshold
