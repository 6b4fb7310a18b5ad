"""Seeded synthetic inputs for the MiniMax-H3-Image DiT block.

This module only draws numbers: weights, latent and text tokens, timesteps and
latent-grid shapes. It holds none of the block's arithmetic, so both the CUDA
path and the CPU oracle can be fed the very same bytes from it without sharing
any of the method.

Recipe (the same on both sides):
  * generator: numpy PCG64 seeded per tensor (seed, tag) so that each tensor is
    reproducible on its own;
  * block linears (QKV, out-projection, FFN, AdaLN): N(0, 0.02), rounded to the
    nearest bf16 (ties to even), because the model card gives the DiT weights
    in BF16 (MiniMax-H3-Image model card, "Model Architecture");
  * timestep MLP: N(0, 0.02) kept in fp32 (the same card: "the embedding,
    timestep and output layers are FP32");
  * biases: zero;
  * tokens: N(0, 1), rounded to bf16;
  * timestep: U[0, 1) drawn from the seed, or given.

Token counts follow the model card's patchification: a 16x VAE downsample and
a 2x2 patch make one token per 32x32 pixels, so a 4096^2 canvas is a 128x128
grid of 16,384 tokens (H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin,
"Inference Optimizations").
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Sequence, Tuple

import numpy as np

PIXELS_PER_TOKEN = 32  # 16x VAE downsample times a 2x2 patch


@dataclasses.dataclass(frozen=True)
class Dims:
    """Model widths of one DiT block."""

    hidden: int
    heads: int
    head_dim: int
    ffn: int
    time_dim: int = 256

    @property
    def inner(self) -> int:
        return self.heads * self.head_dim


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: widths, the packed token layout and a seed."""

    name: str
    dims: Dims
    n_txt: int
    grids: Tuple[Tuple[int, int, int], ...]  # (frame, height, width) per image
    seed: int
    t: float | None  # None: draw from the seed

    @property
    def n_img(self) -> int:
        return sum(h * w for _, h, w in self.grids)

    @property
    def n_tokens(self) -> int:
        return self.n_txt + self.n_img


def canvas_grid(pixels: int) -> int:
    """Latent-grid side for a square canvas side in pixels."""
    if pixels % PIXELS_PER_TOKEN:
        raise ValueError("canvas side must be a multiple of 32 pixels")
    return pixels // PIXELS_PER_TOKEN


SMALL = Dims(hidden=768, heads=8, head_dim=96, ffn=2048)
FULL_96 = Dims(hidden=5376, heads=56, head_dim=96, ffn=14336)
FULL_128 = Dims(hidden=5376, heads=56, head_dim=128, ffn=14336)

_G2K = canvas_grid(2048)  # 64
_G4K = canvas_grid(4096)  # 128

WORKLOADS: Dict[str, Workload] = {
    # one small block: 16x16 latent grid plus 32 text tokens, t = 0.5
    "small_block": Workload("small_block", SMALL, 32, ((0, 16, 16),), 0, 0.5),
    # one full-width block at a 2048^2 canvas plus 512 text tokens
    "block_2k": Workload("block_2k", FULL_96, 512, ((0, _G2K, _G2K),), 0, None),
    "block_2k_dh128": Workload("block_2k_dh128", FULL_128, 512, ((0, _G2K, _G2K),), 0, None),
    # one full-width block at a 4096^2 canvas plus 512 text tokens
    "block_4k": Workload("block_4k", FULL_96, 512, ((0, _G4K, _G4K),), 0, None),
    "block_4k_dh128": Workload("block_4k_dh128", FULL_128, 512, ((0, _G4K, _G4K),), 0, None),
    # reference edit: 2048^2 target plus four 2048^2 references, 256 text tokens
    "edit_4ref": Workload(
        "edit_4ref", FULL_96, 256,
        tuple((k, _G2K, _G2K) for k in range(5)), 0, None),
    "edit_4ref_dh128": Workload(
        "edit_4ref_dh128", FULL_128, 256,
        tuple((k, _G2K, _G2K) for k in range(5)), 0, None),
}

N_BLOCKS = 50
N_STEPS = 6


def _rng(seed: int, tag: str) -> np.random.Generator:
    mix = zlib.crc32(tag.encode()) & 0xFFFFFFFF
    return np.random.Generator(np.random.PCG64([int(seed), mix]))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns of values that are already bf16-representable."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not bf16-representable")
    return (u >> 16).astype(np.uint16)


def bits_to_float(bits: np.ndarray) -> np.ndarray:
    """fp32 values of bf16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape: Sequence[int], std: float, seed: int, tag: str) -> np.ndarray:
    g = _rng(seed, tag)
    return round_to_bf16(g.standard_normal(tuple(shape), dtype=np.float32) * np.float32(std))


def normal_f32(shape: Sequence[int], std: float, seed: int, tag: str) -> np.ndarray:
    g = _rng(seed, tag)
    return (g.standard_normal(tuple(shape), dtype=np.float32) * np.float32(std)).astype(np.float32)


def block_weights(d: Dims, seed: int, std: float = 0.02) -> Dict[str, np.ndarray]:
    """Random-init weights of one block, nn.Linear layout [out, in].

    w_qkv rows are [Q heads | K heads | V heads], each head's head_dim rows
    contiguous; w_ada rows are six chunks of `hidden` rows in the order
    shift1, scale1, gate1, shift2, scale2, gate2.
    """
    D, I, F = d.hidden, d.inner, d.ffn
    return {
        "w_qkv": normal_bf16((3 * I, D), std, seed, "w_qkv"),
        "w_o": normal_bf16((D, I), std, seed, "w_o"),
        "w_ff1": normal_bf16((F, D), std, seed, "w_ff1"),
        "w_ff2": normal_bf16((D, F), std, seed, "w_ff2"),
        "w_ada": normal_bf16((6 * D, D), std, seed, "w_ada"),
        "b_ada": np.zeros((6 * D,), np.float32),
    }


def time_weights(d: Dims, seed: int, std: float = 0.02) -> Dict[str, np.ndarray]:
    """Random-init fp32 timestep MLP: Linear(time_dim -> D), SiLU, Linear(D -> D)."""
    D = d.hidden
    return {
        "w_t1": normal_f32((D, d.time_dim), std, seed, "w_t1"),
        "b_t1": np.zeros((D,), np.float32),
        "w_t2": normal_f32((D, D), std, seed, "w_t2"),
        "b_t2": np.zeros((D,), np.float32),
    }


def tokens(n: int, d: int, seed: int, tag: str) -> np.ndarray:
    return normal_bf16((n, d), 1.0, seed, tag)


def timestep(w: Workload) -> float:
    if w.t is not None:
        return float(w.t)
    return float(_rng(w.seed, "t").random())


def step_timesteps(n_steps: int = N_STEPS) -> List[float]:
    """Timesteps of the sampling loop, 1, 5/6, ..., 1/6 (an assumed schedule:
    the real one ships in a file that is not available)."""
    return [1.0 - k / n_steps for k in range(n_steps)]


def workload_inputs(w: Workload) -> Dict[str, np.ndarray | float]:
    """Text tokens, image tokens and the timestep of a workload."""
    D = w.dims.hidden
    return {
        "x_txt": tokens(w.n_txt, D, w.seed, "x_txt"),
        "x_img": tokens(w.n_img, D, w.seed, "x_img"),
        "t": timestep(w),
    }


def ragged(dims: Dims, n_txt: int, grids: Sequence[Tuple[int, int, int]], seed: int,
           t: float = 0.5, name: str = "ragged") -> Workload:
    """A workload with arbitrary token counts (for tails and edge cases)."""
    return Workload(name, dims, n_txt, tuple(tuple(g) for g in grids), seed, t)


# --- the image VAE's ViT decoder (shape level) --------------------------------
# The same recipe: linears N(0, 0.02) rounded to bf16 (the pages' BF16 decode
# control), their biases and the LayerNorm gains and biases fp32, drawn
# (gains 1 + N(0, 0.1), biases N(0, 0.02)) so that every affine term is
# exercised. Latents N(0, 1) in fp32.

@dataclasses.dataclass(frozen=True)
class VaeDims:
    width: int = 1280
    heads: int = 10
    head_dim: int = 128
    mlp: int = 5120
    layers: int = 24
    tile: int = 32
    channels: int = 24
    out_features: int = 768  # 3 x 16 x 16 pixels per token


VAE = VaeDims()
VAE_SMALL = VaeDims(width=256, heads=2, head_dim=128, mlp=1024, layers=2, tile=16)


def vae_weights(v: VaeDims, seed: int, std: float = 0.02) -> Dict:
    """Random-init decoder weights, nn.Linear layout [out, in]; w_qkv rows are
    [Q heads | K heads | V heads], each head's head_dim rows contiguous."""
    W, M = v.width, v.mlp
    f = lambda shape, tag, s=std: normal_f32(shape, s, seed, tag)
    gain = lambda tag: (1.0 + normal_f32((W,), 0.1, seed, tag)).astype(np.float32)
    layers = []
    for l in range(v.layers):
        t = f"l{l}_"
        layers.append({
            "ln1_g": gain(t + "ln1_g"), "ln1_b": f((W,), t + "ln1_b"),
            "w_qkv": normal_bf16((3 * W, W), std, seed, t + "w_qkv"), "b_qkv": f((3 * W,), t + "b_qkv"),
            "w_o": normal_bf16((W, W), std, seed, t + "w_o"), "b_o": f((W,), t + "b_o"),
            "ln2_g": gain(t + "ln2_g"), "ln2_b": f((W,), t + "ln2_b"),
            "w_1": normal_bf16((M, W), std, seed, t + "w_1"), "b_1": f((M,), t + "b_1"),
            "w_2": normal_bf16((W, M), std, seed, t + "w_2"), "b_2": f((W,), t + "b_2"),
        })
    return {"w_in": normal_f32((W, v.channels), 0.2, seed, "w_in"), "b_in": f((W,), "b_in"),
            "layers": layers, "lnf_g": gain("lnf_g"), "lnf_b": f((W,), "lnf_b"),
            "w_out": normal_bf16((v.out_features, W), std, seed, "w_out"),
            "b_out": f((v.out_features,), "b_out")}
