"""Seeded synthetic inputs for the NVFP4 MoE layer (shared by the tests, the bench
and the oracle's callers).

This module only MAKES DATA. It holds none of the layer's arithmetic: no decoding
of codes or scales, no routing, no projections. It draws BF16 weights and
activations from torch's seeded generators (CPU: Mersenne twister; CUDA: Philox,
so a CPU and a CUDA draw of the same seed differ -- every check feeds one draw to
both sides) and encodes the weights into NVFP4 planes with the quantiser the
tiny-layer workload defines:

    global  = amax(W) / (6 * 448)                   computed in FP64, stored FP32
    scale_g = RNE_E4M3(amax(group of 16) / (6 * global))
    code    = RNE_E2M1(w / (scale_g * global))      ties to the even mantissa

All quantiser arithmetic runs in float64, where every step (the division, the
power-of-two rescales, the threshold compares) is exact or correctly rounded on
both CPU and GPU, so a CPU and a CUDA run encode the same BF16 weights into the
same bytes. The oracle carries an independent FP64 implementation of this
quantiser; a CPU test asserts byte equality between the two.

Workload shapes (the pages' 512-expert, hidden 2048, intermediate 768, top-10
layer; "Strata NVFP4" README and "#2727 ... CSF checkpoint conversion",
"Validation": 512 experts per tensor, 48 layers) are in CONFIGS.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BASE_SEED = 0x4E564650  # "NVFP" in ASCII

# E2M1 magnitudes in code order 0..7 (OCP Microscaling spec, FP4 E2M1 table).
# Used only to pick the rounding thresholds of the encoder below.
_E2M1_TIES_DOWN = (0.25, 1.25, 2.5, 5.0)   # midpoints where the lower neighbour has the even mantissa
_E2M1_TIES_UP = (0.75, 1.75, 3.5)          # midpoints where the upper neighbour has the even mantissa


@dataclass(frozen=True)
class LayerDims:
    E: int
    H: int
    I: int
    K: int


@dataclass(frozen=True)
class Workload:
    name: str
    dims: LayerDims
    tokens: tuple
    act: str = "bf16"          # "bf16" | "int8"
    outliers: bool = False     # 0.1% channels x20
    zipf_s: float | None = None
    layers: int = 1
    seed_index: int = 0
    note: str = ""


TINY = LayerDims(E=8, H=256, I=128, K=2)
BIG = LayerDims(E=512, H=2048, I=768, K=10)

CONFIGS = {
    "tiny": Workload("tiny", TINY, (64,), seed_index=0,
                     note="8 experts, H 256, I 128, top-2, 64 tokens"),
    "decode": Workload("decode", BIG, (1, 2, 4, 8), outliers=True, zipf_s=1.1, seed_index=1,
                       note="512 experts, H 2048, I 768, top-10, T in {1,2,4,8}"),
    "prefill8k": Workload("prefill8k", BIG, (8192,), zipf_s=1.1, seed_index=2,
                          note="512 experts, H 2048, I 768, top-10, 8192-token chunk, BF16"),
    "w4a8_32k": Workload("w4a8_32k", BIG, (32768,), act="int8", outliers=True, zipf_s=1.1,
                         seed_index=3, note="same layer, 32768-token chunk, int8 + per-token scale"),
    "stack48": Workload("stack48", BIG, (1, 2, 4, 4096), zipf_s=1.1, layers=48, seed_index=4,
                        note="48 independently seeded layers, residual carried in FP32"),
}


def _mix(*parts: int) -> int:
    """SplitMix64 finaliser over the parts: a stable 63-bit sub-seed."""
    z = 0x9E3779B97F4A7C15
    for p in parts:
        z = (z + (int(p) & 0xFFFFFFFFFFFFFFFF) + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        z ^= z >> 31
    return z & 0x7FFFFFFFFFFFFFFF


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_mix(*parts))
    return g


def workload_seed(wl: Workload, layer: int = 0) -> int:
    return BASE_SEED + wl.seed_index + layer


# ----------------------------------------------------------------------------
# NVFP4 quantiser (data synthesis only; the layer never quantises weights)
# ----------------------------------------------------------------------------

def _e4m3_encode_rne(v: torch.Tensor) -> torch.Tensor:
    """Non-negative float64 values <= 448 (slightly above is clamped) -> E4M3FN
    bytes, round to nearest, ties to even. Subnormals step 2^-9; normals keep 3
    mantissa bits. A result that rounds up to the next binade carries into the
    exponent field by plain integer addition."""
    v = v.clamp(min=0.0, max=448.0)
    sub = v < 2.0 ** -6
    q_sub = torch.round(v * 512.0)                      # exact scale; round half even
    mant, expo = torch.frexp(torch.where(sub, torch.ones_like(v), v))
    q_norm = torch.round(mant * 16.0)                   # in [8, 16]
    byte_norm = ((expo.to(torch.int64) - 1 + 7) << 3) + (q_norm.to(torch.int64) - 8)
    byte = torch.where(sub, q_sub.to(torch.int64), byte_norm)
    return byte.to(torch.uint8)


def _e4m3_value(byte: torch.Tensor) -> torch.Tensor:
    """Value of non-negative, non-NaN E4M3FN bytes as float64 (the encoder's own
    inverse, needed to form the divisor of the code step)."""
    b = byte.to(torch.int64)
    e = (b >> 3) & 0xF
    m = (b & 0x7).to(torch.float64)
    normal = torch.ldexp(1.0 + m / 8.0, (e - 7).to(torch.float64))
    subn = m * 2.0 ** -9
    return torch.where(e == 0, subn, normal)


def _e2m1_encode_rne(r: torch.Tensor) -> torch.Tensor:
    """float64 ratios -> E2M1 nibbles (sign bit 3), nearest value with ties to the
    even mantissa, saturating at 6."""
    a = r.abs()
    idx = torch.zeros(a.shape, dtype=torch.int64, device=a.device)
    for t in _E2M1_TIES_DOWN:
        idx += (a > t).to(torch.int64)
    for t in _E2M1_TIES_UP:
        idx += (a >= t).to(torch.int64)
    sign = (r < 0).to(torch.int64) << 3
    return (idx | sign).to(torch.uint8)


def quantize_nvfp4(w: torch.Tensor):
    """Quantise BF16 weights of shape [..., rows, cols] (cols % 16 == 0) with one
    global per leading index.

    Returns (codes u8 [..., rows, cols/2], scales u8 [..., rows, cols/16],
    global f32 [...]). Element 2c sits in the low nibble of byte c.
    """
    assert w.dtype == torch.bfloat16 and w.shape[-1] % 16 == 0
    lead = w.shape[:-2]
    rows, cols = w.shape[-2], w.shape[-1]
    w64 = w.to(torch.float64)
    amax = w64.abs().amax(dim=(-2, -1))                              # [...]
    glob32 = (amax / (6.0 * 448.0)).to(torch.float32)
    g64 = glob32.to(torch.float64)
    grp = w64.reshape(*lead, rows, cols // 16, 16)
    gamax = grp.abs().amax(dim=-1)                                   # [..., rows, cols/16]
    gq = g64.reshape(*lead, 1, 1)
    ratio = torch.where(gq > 0, gamax / torch.where(gq > 0, gq, torch.ones_like(gq)) / 6.0,
                        torch.zeros_like(gamax))
    scales = _e4m3_encode_rne(ratio)
    step = _e4m3_value(scales) * gq                                  # exact product in FP64
    step_e = step.unsqueeze(-1)
    r = torch.where(step_e > 0, grp / torch.where(step_e > 0, step_e, torch.ones_like(step_e)),
                    torch.zeros_like(grp))
    nib = _e2m1_encode_rne(r).reshape(*lead, rows, cols)
    codes = (nib[..., 0::2] | (nib[..., 1::2] << 4)).contiguous()
    return codes, scales.contiguous(), glob32.contiguous()


# ----------------------------------------------------------------------------
# Layers, activations, router logits
# ----------------------------------------------------------------------------

@dataclass
class Layer:
    dims: LayerDims
    gate_codes: torch.Tensor
    up_codes: torch.Tensor
    gate_scales: torch.Tensor
    up_scales: torch.Tensor
    gate_global: torch.Tensor
    up_global: torch.Tensor
    down_codes: torch.Tensor
    down_scales: torch.Tensor
    down_global: torch.Tensor
    bf16: dict = field(default_factory=dict)   # the BF16 weights, when kept

    def planes(self):
        return (self.gate_codes, self.up_codes, self.gate_scales, self.up_scales,
                self.gate_global, self.up_global, self.down_codes, self.down_scales,
                self.down_global)

    def to(self, device):
        kw = {k: getattr(self, k).to(device) for k in (
            "gate_codes", "up_codes", "gate_scales", "up_scales", "gate_global",
            "up_global", "down_codes", "down_scales", "down_global")}
        return Layer(self.dims, **kw)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.planes())


EXPERT_BATCH = 8  # experts drawn per generator call (part of the recipe: fixes the stream)


def make_layer(dims: LayerDims, seed: int, device="cpu", std: float = 0.02,
               keep_bf16: bool = False) -> Layer:
    """Weights ~ BF16(N(0, std^2)), one generator stream per projection, drawn
    EXPERT_BATCH experts at a time, then quantised per (expert, projection)."""
    E, H, I = dims.E, dims.H, dims.I
    u8 = dict(dtype=torch.uint8, device=device)
    out = {
        "gate_codes": torch.empty(E, I, H // 2, **u8), "gate_scales": torch.empty(E, I, H // 16, **u8),
        "up_codes": torch.empty(E, I, H // 2, **u8), "up_scales": torch.empty(E, I, H // 16, **u8),
        "down_codes": torch.empty(E, H, I // 2, **u8), "down_scales": torch.empty(E, H, I // 16, **u8),
        "gate_global": torch.empty(E, dtype=torch.float32, device=device),
        "up_global": torch.empty(E, dtype=torch.float32, device=device),
        "down_global": torch.empty(E, dtype=torch.float32, device=device),
    }
    kept = {}
    for pi, (name, rows, cols) in enumerate((("gate", I, H), ("up", I, H), ("down", H, I))):
        g = _gen(device, seed, 101, pi)
        for e0 in range(0, E, EXPERT_BATCH):
            eb = min(EXPERT_BATCH, E - e0)
            w = (torch.randn(eb, rows, cols, generator=g, device=device, dtype=torch.float32)
                 * std).to(torch.bfloat16)
            c, s, gl = quantize_nvfp4(w)
            out[f"{name}_codes"][e0:e0 + eb] = c
            out[f"{name}_scales"][e0:e0 + eb] = s
            out[f"{name}_global"][e0:e0 + eb] = gl
            if keep_bf16:
                kept.setdefault(name, []).append(w)
    layer = Layer(dims, **out)
    if keep_bf16:
        layer.bf16 = {k: torch.cat(v) for k, v in kept.items()}
    return layer


def outlier_channels(H: int, seed: int, device="cpu") -> torch.Tensor:
    n = max(1, round(0.001 * H))
    g = _gen("cpu", seed, 202)
    return torch.randperm(H, generator=g)[:n].to(device)


def make_x_f32(T: int, H: int, seed: int, outliers: bool, device="cpu") -> torch.Tensor:
    """N(0,1) activations, optionally with 0.1% of channels (round(0.001 H))
    multiplied by 20 for every token."""
    g = _gen(device, seed, 201)
    x = torch.randn(T, H, generator=g, device=device, dtype=torch.float32)
    if outliers:
        ch = outlier_channels(H, seed, device)
        x[:, ch] *= 20.0
    return x


def make_x_bf16(T: int, H: int, seed: int, outliers: bool = False, device="cpu") -> torch.Tensor:
    return make_x_f32(T, H, seed, outliers, device).to(torch.bfloat16)


def make_x_int8(T: int, H: int, seed: int, outliers: bool = True, device="cpu"):
    """Symmetric per-token int8: scale_t = amax_t / 127 (FP32), q = RNE(x/scale)
    clamped to +-127. Returns (q int8 [T][H], scale f32 [T])."""
    x = make_x_f32(T, H, seed, outliers, device)
    amax = x.abs().amax(dim=1)
    scale = amax / 127.0
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    q = torch.round(x / safe[:, None]).clamp(-127, 127).to(torch.int8)
    return q, scale.contiguous()


def zipf_bias(E: int, s: float, seed: int) -> torch.Tensor:
    """bias_e = ln p_{rank(e)}, p_r proportional to r^-s, rank a seeded
    permutation of 1..E. FP64 then rounded to FP32."""
    g = _gen("cpu", seed, 303)
    rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    logp = -s * torch.log(rank)
    logp = logp - torch.logsumexp(logp, dim=0)
    return logp.to(torch.float32)


def make_logits(T: int, E: int, seed: int, zipf_s: float | None = None, device="cpu") -> torch.Tensor:
    g = _gen(device, seed, 301)
    l = torch.randn(T, E, generator=g, device=device, dtype=torch.float32)
    if zipf_s is not None:
        l = l + zipf_bias(E, zipf_s, seed).to(device)
    return l.contiguous()


def make_router_w(E: int, H: int, seed: int, std: float = 0.05, device="cpu") -> torch.Tensor:
    """Router projection weights [E][H] bf16 ~ BF16(N(0, std^2)), one seeded stream."""
    g = _gen(device, seed, 0x52)
    return (torch.randn(E, H, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def make_topk(T: int, E: int, K: int, seed: int, device="cpu"):
    """Precomputed routing: K distinct ids per token drawn uniformly, weights a
    random positive vector normalised to 1 (FP32)."""
    g = _gen("cpu", seed, 401)
    ids = torch.argsort(torch.rand(T, E, generator=g), dim=1)[:, :K].to(torch.int32)
    w = torch.rand(T, K, generator=g, dtype=torch.float64) + 0.05
    w = (w / w.sum(dim=1, keepdim=True)).to(torch.float32)
    return ids.contiguous().to(device), w.contiguous().to(device)
