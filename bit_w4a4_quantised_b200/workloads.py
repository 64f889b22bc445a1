"""Seeded synthetic layer inputs shaped like the Fast-WAM experts.

This module draws inputs only: activations x, weights W, smoothing vector s,
basis V and bias.  It holds none of the layer's arithmetic (no Hadamard, no
deflation, no quantiser), so both the CUDA path and the float64 oracle can take
their inputs from it without sharing any computation.

Shapes follow the layer set the model card quantises ("FastWAM UR3 3-task —
4-bit quantisations", the paragraph under the top table: two experts x 30
blocks x {self-attn q/k/v/o, cross-attn q/k/v/o, ffn.0, ffn.2}).  The real
calibration data and checkpoint are not available, so every tensor is drawn
from a seeded generator:

* RNG: NumPy PCG64 seeded by ``SeedSequence([seed, config_id, layer])``;
  draw order x, outlier channel indices, W, bias, V-Gaussian.
* x: N(0, 1) with a few whole input channels (columns) scaled up as outliers,
  the count rounded to nearest (1 % of 1024 -> 10, 0.5 % of 3072 -> 15,
  0.5 % of 14336 -> 72), channels drawn without replacement.  The FFN-down
  input is GELU (exact erf form) of such a matrix.
* W: N(0, 0.02); bias: N(0, 0.01).  x, W and bias are rounded to bf16
  (round to nearest even) and returned as the float32 values of those bf16
  numbers, so the oracle and the device see identical inputs.
* s: SmoothQuant-style alpha = 0.5, s_j = sqrt(max_m |x_mj|) / sqrt(max_n |W_nj|)
  with both maxima clamped to >= 1e-5, computed in float64, stored fp32.
* V: Q factor of the QR decomposition of a seeded N(0, 1) [K, r] matrix,
  stored fp32 (orthonormal columns up to fp32 rounding).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


def bf16_round(a) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even) and return the
    float32 values of the results.  Inputs must be finite."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(a) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exact bf16 numbers."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not exact bf16 numbers")
    return (u >> 16).astype(np.uint16)


@dataclasses.dataclass
class LayerCase:
    """One linear layer's inputs.  All arrays are float32; x, W and bias hold
    exact bf16 values."""

    name: str
    M: int
    K: int
    N: int
    r: int
    b: int
    x: np.ndarray      # [M, K]
    W: np.ndarray      # [N, K]
    s: np.ndarray      # [K]
    V: np.ndarray      # [K, r]
    bias: np.ndarray   # [N]

    @property
    def shape(self) -> tuple[int, int, int]:
        return self.M, self.K, self.N


def _rng(seed: int, config_id: int, layer: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, config_id, layer])))


def _gelu_erf(v: np.ndarray) -> np.ndarray:
    from scipy.special import erf
    v64 = v.astype(np.float64)
    return (0.5 * v64 * (1.0 + erf(v64 / math.sqrt(2.0)))).astype(np.float32)


def smoothing_vector(x: np.ndarray, W: np.ndarray, clamp: float = 1e-5) -> np.ndarray:
    """alpha = 0.5 smoothing vector from the same x and W (input recipe)."""
    ax = np.maximum(np.abs(x.astype(np.float64)).max(axis=0), clamp)
    aw = np.maximum(np.abs(W.astype(np.float64)).max(axis=0), clamp)
    return (np.sqrt(ax) / np.sqrt(aw)).astype(np.float32)


def draw_layer(name: str, M: int, K: int, N: int, r: int, b: int, *,
               seed: int, config_id: int, layer: int = 0,
               n_outliers: int = 0, outlier_scale: float = 1.0,
               gelu_input: bool = False, w_std: float = 0.02,
               bias_std: float = 0.01, v_rank: int | None = None) -> LayerCase:
    """Draw one layer in the documented order.  ``v_rank`` lets r = 0 and
    r = 32 variants share x, W and bias (V is drawn with v_rank columns and
    cut to r)."""
    rng = _rng(seed, config_id, layer)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if n_outliers:
        idx = rng.choice(K, size=n_outliers, replace=False)
        x[:, idx] *= np.float32(outlier_scale)
    if gelu_input:
        x = _gelu_erf(x)
    x = bf16_round(x)
    W = bf16_round(rng.standard_normal((N, K), dtype=np.float32) * np.float32(w_std))
    bias = bf16_round(rng.standard_normal(N, dtype=np.float32) * np.float32(bias_std))
    vr = r if v_rank is None else v_rank
    if vr:
        G = rng.standard_normal((K, vr))
        Q, _ = np.linalg.qr(G)
        V = Q[:, :r].astype(np.float32)
    else:
        V = np.zeros((K, 0), dtype=np.float32)
    s = smoothing_vector(x, W)
    return LayerCase(name, M, K, N, r, b, x, W, s, np.ascontiguousarray(V), bias)


def outlier_count(K: int, frac: float) -> int:
    return int(math.floor(K * frac + 0.5))


# ---------------------------------------------------------------------------
# The five workloads.
# ---------------------------------------------------------------------------

def c1_tiny(seed: int = 0) -> LayerCase:
    """Single tiny ASP layer: x [64, 256] with 4 outlier channels x20,
    W [256, 256], Hadamard block 16, rank 32."""
    return draw_layer("c1_tiny_64x256x256_r32_b16", 64, 256, 256, 32, 16, seed=seed,
                      config_id=1, n_outliers=4, outlier_scale=20.0)


def c2_action_attn(seed: int = 0, layer: int = 0) -> LayerCase:
    """Action-expert attention projection: 32 tokens, 1024 -> 1024, rank 32,
    block 128, 1 % outlier channels x20 (small-M, weight streaming)."""
    return draw_layer("c2_action_attn_32x1024x1024_r32_b128", 32, 1024, 1024, 32, 128,
                      seed=seed, config_id=2, layer=layer,
                      n_outliers=outlier_count(1024, 0.01), outlier_scale=20.0)


def c3_video_attn(r: int = 32, seed: int = 0, layer: int = 0) -> LayerCase:
    """Video-expert attention projection: 4096 tokens, 3072 -> 3072, block 128,
    0.5 % outlier channels x30; r = 0 and r = 32 share x, W and bias."""
    return draw_layer(f"c3_video_attn_4096x3072x3072_r{r}_b128", 4096, 3072, 3072, r, 128,
                      seed=seed, config_id=3, layer=layer,
                      n_outliers=outlier_count(3072, 0.005), outlier_scale=30.0, v_rank=32)


def c3_video_attn_int4(seed: int = 0, layer: int = 0) -> LayerCase:
    """The c3 layer (same x, W, bias and V as c3_video_attn(32)) for the
    SVDQuant INT4 arm: no rotation (block 1), rank 32."""
    return draw_layer("c3_video_attn_4096x3072x3072_r32_b1", 4096, 3072, 3072, 32, 1,
                      seed=seed, config_id=3, layer=layer,
                      n_outliers=outlier_count(3072, 0.005), outlier_scale=30.0, v_rank=32)


def c2_action_attn_int4(seed: int = 0, layer: int = 0) -> LayerCase:
    """The c2 layer (same draws as c2_action_attn) for the SVDQuant INT4 arm:
    block 1, rank 32."""
    return draw_layer("c2_action_attn_32x1024x1024_r32_b1", 32, 1024, 1024, 32, 1,
                      seed=seed, config_id=2, layer=layer,
                      n_outliers=outlier_count(1024, 0.01), outlier_scale=20.0)


def c4_video_ffn_up(seed: int = 0) -> LayerCase:
    """Video-expert FFN up: 4096 tokens, 3072 -> 14336, rank 32, block 128."""
    return draw_layer("c4_video_ffn_up_4096x3072x14336_r32_b128", 4096, 3072, 14336, 32, 128,
                      seed=seed, config_id=4, layer=0,
                      n_outliers=outlier_count(3072, 0.005), outlier_scale=30.0)


def c4_video_ffn_down(seed: int = 0) -> LayerCase:
    """Video-expert FFN down: input GELU(Gaussian with 72 outlier channels x30),
    4096 tokens, 14336 -> 3072, rank 32, block 128."""
    return draw_layer("c4_video_ffn_down_4096x14336x3072_r32_b128", 4096, 14336, 3072, 32, 128,
                      seed=seed, config_id=4, layer=1,
                      n_outliers=outlier_count(14336, 0.005), outlier_scale=30.0,
                      gelu_input=True)


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    r: int


def c5_layer_specs(cross_kv_context: bool = True) -> list[LayerSpec]:
    """The 600 linears of one denoising step of the 2-expert MoT.

    Video expert: d = 3072, ffn 14336, 4096 tokens, r = 0.  Action expert:
    d = 1024, ffn 4096, 32 tokens, r = 32; with ``cross_kv_context`` its
    cross-attention k/v projections read the 4096-token context (the literal
    reading of "cross-attn K from M=4096 context")."""
    specs = []
    for blk in range(30):
        dv, fv, Mv = 3072, 14336, 4096
        for p in ("self_q", "self_k", "self_v", "self_o",
                  "cross_q", "cross_k", "cross_v", "cross_o"):
            specs.append(LayerSpec(f"video.{blk}.{p}", Mv, dv, dv, 0))
        specs.append(LayerSpec(f"video.{blk}.ffn0", Mv, dv, fv, 0))
        specs.append(LayerSpec(f"video.{blk}.ffn2", Mv, fv, dv, 0))
    for blk in range(30):
        da, fa, Ma = 1024, 4096, 32
        for p in ("self_q", "self_k", "self_v", "self_o", "cross_q", "cross_o"):
            specs.append(LayerSpec(f"action.{blk}.{p}", Ma, da, da, 32))
        Mkv = 4096 if cross_kv_context else Ma
        specs.append(LayerSpec(f"action.{blk}.cross_k", Mkv, da, da, 32))
        specs.append(LayerSpec(f"action.{blk}.cross_v", Mkv, da, da, 32))
        specs.append(LayerSpec(f"action.{blk}.ffn0", Ma, da, fa, 32))
        specs.append(LayerSpec(f"action.{blk}.ffn2", Ma, fa, da, 32))
    return specs


def c5_layer(index: int, seed: int = 0, cross_kv_context: bool = True) -> LayerCase:
    """Draw layer ``index`` of the C5 step (block 128, outliers as C3)."""
    spec = c5_layer_specs(cross_kv_context)[index]
    frac, scale = (0.005, 30.0) if spec.name.startswith("video") else (0.01, 20.0)
    return draw_layer(spec.name, spec.M, spec.K, spec.N, spec.r, 128, seed=seed,
                      config_id=5, layer=index,
                      n_outliers=outlier_count(spec.K, frac), outlier_scale=scale)


def custom(M: int, K: int, N: int, r: int, b: int, seed: int = 0, layer: int = 0,
           n_outliers: int = 0, outlier_scale: float = 20.0) -> LayerCase:
    """Any shape, for parity sweeps (config id 99)."""
    return draw_layer(f"custom_{M}x{K}x{N}_r{r}_b{b}", M, K, N, r, b, seed=seed,
                      config_id=99, layer=layer, n_outliers=n_outliers,
                      outlier_scale=outlier_scale)


WORKLOADS = {
    "c1": c1_tiny,
    "c2": c2_action_attn,
    "c3r0": lambda seed=0: c3_video_attn(0, seed),
    "c3": lambda seed=0: c3_video_attn(32, seed),
    "c4up": c4_video_ffn_up,
    "c4down": c4_video_ffn_down,
}


# ---------------------------------------------------------------------------
# The same recipe drawn on the device (benchmark inputs too large to draw on
# the host in a few minutes: the 600 linears of one denoising step hold 5.4 B
# weights).  torch's CUDA generator (Philox) replaces PCG64, so the values
# differ from the NumPy draws of the same (seed, config, layer); the
# distributions, the draw order and the derived s and V follow the recipe
# above.  Parity tests use the NumPy draws.
# ---------------------------------------------------------------------------

def _device_generator(device, seed: int, config_id: int, layer: int):
    import torch
    key = np.random.SeedSequence([seed, config_id, layer]).generate_state(2, dtype=np.uint64)
    g = torch.Generator(device=device)
    g.manual_seed(int(key[0] & np.uint64(0x7FFFFFFFFFFFFFFF)))
    return g


def draw_layer_device(spec: LayerSpec, *, seed: int, config_id: int, layer: int, device, b: int = 128,
                      n_outliers: int = 0, outlier_scale: float = 1.0, w_std: float = 0.02,
                      bias_std: float = 0.01) -> dict:
    """One layer's inputs as device tensors: x, W, bias bf16; s, V fp32 (V is
    None for r = 0).  Returns a dict with the spec's M, K, N, r and b."""
    import torch
    g = _device_generator(device, seed, config_id, layer)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if n_outliers:
        idx = torch.randperm(K, generator=g, device=device)[:n_outliers]
        x[:, idx] *= outlier_scale
    x = x.to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * w_std).to(torch.bfloat16)
    bias = (torch.randn((N,), generator=g, device=device, dtype=torch.float32) * bias_std).to(torch.bfloat16)
    V = None
    if r:
        G = torch.randn((K, r), generator=g, device=device, dtype=torch.float64)
        V = torch.linalg.qr(G)[0].to(torch.float32).contiguous()
    ax = x.abs().amax(dim=0).to(torch.float64).clamp_min(1e-5)
    aw = W.abs().amax(dim=0).to(torch.float64).clamp_min(1e-5)
    s = (ax.sqrt() / aw.sqrt()).to(torch.float32).contiguous()
    return {"M": M, "K": K, "N": N, "r": r, "b": b, "x": x, "W": W, "bias": bias, "s": s, "V": V}


def c5_layer_device(index: int, device, seed: int = 0, cross_kv_context: bool = True) -> dict:
    """Layer ``index`` of the C5 step drawn on the device (outliers as c5_layer)."""
    spec = c5_layer_specs(cross_kv_context)[index]
    frac, scale = (0.005, 30.0) if spec.name.startswith("video") else (0.01, 20.0)
    d = draw_layer_device(spec, seed=seed, config_id=5, layer=index, device=device,
                          n_outliers=outlier_count(spec.K, frac), outlier_scale=scale)
    d["name"] = spec.name
    return d
