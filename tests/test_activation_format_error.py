"""How far the layer moves when its activations are quantised the way a
block-scaled FP4 x FP4 prompt path (tcgen05 `kind::mxf4nvf4`) or the W4A8 path
needs them -- the accuracy half of the choice between block-scaled MMA and exact
dequantisation ("Strata NVFP4" README, "How it differs from upstream Strata", the
W4A8 bullet: 8-bit activations err far less per product than FP4 ones).

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
