"""Brute-force dense formulation of the MoE layer -- TEST INFRASTRUCTURE, used only
to pin the C oracle on tiny layers.

It is a different algorithm from the oracle: every expert's matrices are decoded
to dense FP64 arrays with numpy/torch library conversions (torch.float8_e4m3fn
for the scales, a table of the OCP MX E2M1 magnitudes for the codes, a bit shift
for BF16), routing is a dense [T][E] gate matrix built from a library sort and a
library softmax, and the layer is evaluated for ALL experts as matrix products:

    out = sum_e  gate[:, e] * ( s_d(e) * SwiGLU(s_g(e) X G_e^T, s_u(e) X U_e^T) D_e^T )
"""
from __future__ import annotations

import numpy as np
import torch

# OCP Microscaling spec, FP4 E2M1 table: magnitudes of codes 0..7.
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _t(a):
    return a.detach().cpu() if hasattr(a, "detach") else torch.from_numpy(np.ascontiguousarray(a))


def dense(codes, scales, glob) -> np.ndarray:
    """[rows][cols/2] codes, [rows][cols/16] scales, scalar glob -> FP64 [rows][cols]."""
    c = _t(codes).to(torch.int64)
    lo, hi = c & 0xF, c >> 4
    nib = torch.stack([lo, hi], dim=-1).reshape(c.shape[0], -1)
    mag = torch.tensor(E2M1_MAGNITUDES, dtype=torch.float64)[nib & 7]
    val = torch.where((nib & 8) != 0, -mag, mag)
    s = _t(scales).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    s = s.repeat_interleave(16, dim=1)
    return (val * s * float(glob)).numpy()


def bf16_to_f64(x) -> np.ndarray:
    xt = _t(x)
    if xt.dtype == torch.bfloat16:
        return xt.to(torch.float64).numpy()
    bits = xt.view(torch.int16).to(torch.int32) & 0xFFFF
    return (bits << 16).to(torch.int32).view(torch.float32).to(torch.float64).numpy()


def gate_matrix(logits, K: int) -> np.ndarray:
    """Dense [T][E] routing weights: top-K by a stable library sort on (-logit, id),
    softmax (library) over the selected logits."""
    l = np.asarray(_t(logits).to(torch.float64).numpy())
    T, E = l.shape
    G = np.zeros((T, E))
    for t in range(T):
        order = np.lexsort((np.arange(E), -l[t]))[:K]
        sel = torch.softmax(torch.from_numpy(l[t, order]), dim=0).numpy()
        G[t, order] = sel
    return G


def gate_matrix_from(ids, wts, E: int) -> np.ndarray:
    ids = np.asarray(_t(ids).numpy())
    w = np.asarray(_t(wts).to(torch.float64).numpy())
    G = np.zeros((ids.shape[0], E))
    for t in range(ids.shape[0]):
        G[t, ids[t]] = w[t]
    return G


def layer_out(layer, X: np.ndarray, G: np.ndarray) -> np.ndarray:
    """X: FP64 [T][H] activations (already scaled), G: dense [T][E] gate."""
    E = G.shape[1]
    out = np.zeros((X.shape[0], layer.down_codes.shape[1]))
    for e in range(E):
        if not np.any(G[:, e]):
            continue
        Wg = dense(layer.gate_codes[e], layer.gate_scales[e], layer.gate_global[e])
        Wu = dense(layer.up_codes[e], layer.up_scales[e], layer.up_global[e])
        Wd = dense(layer.down_codes[e], layer.down_scales[e], layer.down_global[e])
        g = X @ Wg.T
        u = X @ Wu.T
        h = g * torch.sigmoid(torch.from_numpy(g)).numpy() * u
        y = h @ Wd.T
        out += G[:, e:e + 1] * y
    return out
