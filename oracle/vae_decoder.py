"""Oracle: the image VAE's 2-D ViT decoder, shape level, in float64 on the CPU.

TEST INFRASTRUCTURE, like dit_block.py: only the tests, the smoke check and
the benchmark's CPU-baseline legs import it; it shares no code with the CUDA
library and the library never calls it.

What the pages fix:
  [card] MiniMax-H3-Image model card, "Model Architecture": the image VAE is a
         CNN encoder and a 2D ViT decoder with 24 layers, 16x spatial
         downsampling and 24 latent channels; the VAE is FP32.
  [vllm] "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Faster
         Decoding": the VAE decodes independent image tiles (spread over GPUs,
         with CUDA graphs and streams); a BF16 control is reported.
  [recipe] vLLM-Omni recipe, component table: the VAE has 0.58B parameters.

Readings where the pages are silent (each listed in the design notes; the
decoder runs on random weights, so these fix its shape and cost, not its
numbers):
  V1 layer: a pre-norm ViT block, x += Attn(LN1(x)), x += MLP(LN2(x)); LayerNorm
     with gain and bias, eps 1e-6; every linear has a bias; MLP W -> 4W -> W
     with the exact erf GELU; attention softmax(Q K^T / sqrt(d)) V over the
     tokens of one tile, no mask, no rotary embedding.
  V2 widths: W = 1280, 10 heads x 128, MLP 5120 (24 layers come to 0.47B
     parameters, which with a CNN encoder is in line with the 0.58B total).
  V3 input: one token per latent pixel, Linear(24 -> W) + bias, plus a fixed
     2-D sin-cos position table over the tile's grid (below).
  V4 output: a final LayerNorm, Linear(W -> 3 x 16 x 16) + bias; a token's
     768 outputs are its 16 x 16 RGB pixel block, feature ch*256 + 16 i + j at
     pixel (16 r + i, 16 c + j) of channel ch.
  V5 tiles: the latent is cut into non-overlapping T x T tiles (T = 32 latent
     pixels, 512 image pixels), from the top-left; where a side is not a
     multiple of T the last tiles of that row or column are smaller. Each tile
     is decoded on its own ("independent tiles") and its pixels written at its
     place; nothing is blended.
  V6 position table: indexed by the position inside the tile. The first W/2
     channels encode the row r, the last W/2 the column c, each as
     [sin(p w_k) for k < W/4] followed by [cos(p w_k) for k < W/4], with
     w_k = 10000^(-k / (W/4)).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Sequence

import numpy as np
from scipy.special import erf as _erf

LATENT_CHANNELS = 24
SCALE = 16  # image pixels per latent pixel along each side


@dataclasses.dataclass(frozen=True)
class VaeConfig:
    width: int = 1280
    heads: int = 10
    head_dim: int = 128
    mlp: int = 5120
    layers: int = 24
    tile: int = 32
    channels: int = LATENT_CHANNELS
    eps: float = 1e-6

    @property
    def out_features(self) -> int:
        return 3 * SCALE * SCALE


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def layer_norm(x, gain, bias, eps: float) -> np.ndarray:
    """(x - mean) / sqrt(var + eps) * gain + bias over the last axis (the
    biased variance, as LayerNorm defines it)."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(gain) + _f64(bias)


def gelu(x) -> np.ndarray:
    x = _f64(x)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def affine(x, w, b) -> np.ndarray:
    """x W^T + b for an nn.Linear weight [out, in]."""
    return _f64(x) @ _f64(w).T + _f64(b)


def position_table(h: int, w: int, width: int) -> np.ndarray:
    """V6: [h w, width] sin-cos table of the row-major positions of an h x w
    grid."""
    q = width // 4
    omega = 10000.0 ** (-np.arange(q, dtype=np.float64) / q)
    r, c = np.meshgrid(np.arange(h, dtype=np.float64), np.arange(w, dtype=np.float64),
                       indexing="ij")
    r, c = r.reshape(-1, 1) * omega, c.reshape(-1, 1) * omega
    return np.concatenate([np.sin(r), np.cos(r), np.sin(c), np.cos(c)], axis=1)


def attention(q, k, v) -> np.ndarray:
    """Per head: softmax(Q K^T / sqrt(d)) V over all tokens, q/k/v [n, H, d]."""
    d = q.shape[-1]
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        s = (q[:, h] @ k[:, h].T) / math.sqrt(d)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[:, h] = (p / p.sum(axis=1, keepdims=True)) @ v[:, h]
    return out


def vit_layer(x, w: Dict[str, np.ndarray], cfg: VaeConfig) -> np.ndarray:
    """V1 on one tile's tokens x [n, W]:
        a = LN1(x);  Q|K|V = a W_qkv^T + b_qkv;  x = x + Attn(Q, K, V) W_o^T + b_o
        m = LN2(x);  x = x + GELU(m W_1^T + b_1) W_2^T + b_2
    W_qkv rows are [Q heads | K heads | V heads], each head's d rows contiguous."""
    x = _f64(x)
    n, W = x.shape
    H, d = cfg.heads, cfg.head_dim
    a = layer_norm(x, w["ln1_g"], w["ln1_b"], cfg.eps)
    qkv = affine(a, w["w_qkv"], w["b_qkv"])
    q = qkv[:, :H * d].reshape(n, H, d)
    k = qkv[:, H * d:2 * H * d].reshape(n, H, d)
    v = qkv[:, 2 * H * d:].reshape(n, H, d)
    x = x + affine(attention(q, k, v).reshape(n, H * d), w["w_o"], w["b_o"])
    m = layer_norm(x, w["ln2_g"], w["ln2_b"], cfg.eps)
    return x + affine(gelu(affine(m, w["w_1"], w["b_1"])), w["w_2"], w["b_2"])


def tiles(h: int, w: int, t: int) -> List[tuple]:
    """V5: (row0, col0, rows, cols) of each tile, row-major over the tile grid."""
    out = []
    for r0 in range(0, h, t):
        for c0 in range(0, w, t):
            out.append((r0, c0, min(t, h - r0), min(t, w - c0)))
    return out


def decode_tile(z, weights: Dict, cfg: VaeConfig) -> np.ndarray:
    """One tile's latent z [C, h, w] -> pixels [3, 16 h, 16 w] (V3, V1 x layers, V4)."""
    z = _f64(z)
    C, h, w = z.shape
    x = affine(z.reshape(C, h * w).T, weights["w_in"], weights["b_in"])
    x = x + position_table(h, w, cfg.width)
    for layer in weights["layers"]:
        x = vit_layer(x, layer, cfg)
    y = affine(layer_norm(x, weights["lnf_g"], weights["lnf_b"], cfg.eps),
               weights["w_out"], weights["b_out"])
    return unpatchify_pixels(y, h, w)


def unpatchify_pixels(y, h: int, w: int) -> np.ndarray:
    """Tokens [h w, 3 * 16 * 16] -> pixels [3, 16 h, 16 w] (V4's feature order)."""
    y = _f64(y).reshape(h, w, 3, SCALE, SCALE)            # r, c, ch, i, j
    return y.transpose(2, 0, 3, 1, 4).reshape(3, h * SCALE, w * SCALE)


def decode(z, weights: Dict, cfg: VaeConfig) -> np.ndarray:
    """The latent [C, Hl, Wl] decoded tile by tile (V5) -> image [3, 16 Hl, 16 Wl]."""
    z = _f64(z)
    C, Hl, Wl = z.shape
    img = np.empty((3, Hl * SCALE, Wl * SCALE))
    for r0, c0, h, w in tiles(Hl, Wl, cfg.tile):
        img[:, r0 * SCALE:(r0 + h) * SCALE, c0 * SCALE:(c0 + w) * SCALE] = \
            decode_tile(z[:, r0:r0 + h, c0:c0 + w], weights, cfg)
    return img


def decode_flops(Hl: int, Wl: int, cfg: VaeConfig) -> int:
    """Algorithmic flops of a decode: per token 2 (C W + 3 W^2 + W^2 + 2 W M)
    per layer-linear set and 2 W 768 + 2 C W at the ends, plus 4 n^2 W per
    tile and layer for the attention (no causal halving)."""
    W, M, L = cfg.width, cfg.mlp, cfg.layers
    n_tok = Hl * Wl
    lin = n_tok * (2 * cfg.channels * W + L * 2 * (4 * W * W + 2 * W * M) + 2 * W * cfg.out_features)
    att = sum(L * 4 * (h * w) ** 2 * W for _, _, h, w in tiles(Hl, Wl, cfg.tile))
    return lin + att
