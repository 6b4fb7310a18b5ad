"""Oracle: the MiniMax-H3-Image dense DiT block written out in float64 on the CPU.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module. It shares no code with the CUDA library
and the library never calls it: it is the slow, obviously correct definition
the GPU path is checked against.

Every function computes its result in float64 straight from the definition,
with numpy's matmul as the only library primitive, and no blocking, fusion or
reordering beyond what the definition states.

Sources (page titles; the block as those pages describe it):
  [card]  MiniMax-H3-Image model card (taim.plus mirror of unsloth/MiniMax-H3-Image-FP8),
          "Model Architecture": one packed sequence of text and image tokens
          through a single-stream transformer; 50 layers, hidden 5376, 56 heads,
          FFN 14336; "3D multimodal RoPE"; BF16 weights with the timestep
          layers in FP32.
  [apx]   apxml "MiniMax H3 Image", "Architecture Diagram": per block
          AdaLN modulation (RMSNorm, timestep scale/shift) -> joint attention
          (56 Q / 56 KV heads, head dim 128) -> "+" -> AdaLN modulation
          (RMSNorm, timestep scale/shift) -> GELU MLP (14.3k) -> "+";
          "Specifications": RoPE, RMS normalization, GELU.
  [news]  aib.vote "MiniMax Releases H3 Image Model": 33.1B params, 50 layers,
          hidden 5376, 56 heads, FFN 14336; 6 sampling steps.
  [vllm]  "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin",
          "Inference Optimizations" / "Faster DiT": AdaLN caching (the
          conditioning projection is reused); 16,384 target tokens at 4096^2.

Readings where the pages are silent (each listed in the design notes):
  head_dim is a parameter (96 = 5376/56 from [card]/[news], 128 from [apx]);
  GELU is the exact erf form (tanh form behind a flag); the FFN is not gated;
  the block linears have no bias; RMSNorm has eps 1e-6 and no gain; AdaLN uses
  (1 + scale), + shift and a per-branch gate, six chunks in the order
  shift1, scale1, gate1, shift2, scale2, gate2, projected per block from
  SiLU(c) where c is the timestep MLP output; the timestep sinusoid has 256
  channels [cos | sin] with frequencies 10000^(-i/128) at argument 1000*t;
  RoPE splits head_dim/2 rotation pairs into (frame, row, col) sections,
  each a rotate-half 1-D RoPE over its own contiguous 2*s channels with
  frequencies theta^(-j/s), theta 10000; text tokens sit at position (0,0,0);
  reference image k is frame k; attention is bidirectional, unmasked, scaled
  by 1/sqrt(head_dim). Around the block loop: 2x2 patches of the 24-channel
  latent in pixel-unshuffle order, an FP32 Linear(96 -> D) embedding with
  bias, a DiT output layer (RMSNorm, AdaLN shift/scale, Linear(D -> 96) with
  bias) predicting the flow velocity, and Euler steps from t = 1 to t = 0.

Parity pins: tests/test_oracle_pins.py, and tests/test_oracle_c.py against the
independent C oracle (oracle/h3ref.c). The real model's numbers are "parity
unpinned" (no trained weights or printed activations exist to compare with).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np
from scipy.special import erf as _erf


@dataclasses.dataclass(frozen=True)
class BlockConfig:
    hidden: int
    heads: int
    head_dim: int
    ffn: int
    rope_sections: Tuple[int, int, int]
    rope_theta: float = 10000.0
    norm_eps: float = 1e-6
    t_scale: float = 1000.0
    time_dim: int = 256
    gelu_tanh: bool = False

    @property
    def inner(self) -> int:
        return self.heads * self.head_dim


def default_sections(head_dim: int) -> Tuple[int, int, int]:
    """Rotation pairs per (frame, row, col) axis: (16,16,16) for head_dim 96,
    (16,24,24) for 128. A reading: [card] names "3D multimodal RoPE" but no split."""
    if head_dim == 96:
        return (16, 16, 16)
    if head_dim == 128:
        return (16, 24, 24)
    raise ValueError("head_dim must be 96 or 128")


def config_for(hidden: int, heads: int, head_dim: int, ffn: int, **kw) -> BlockConfig:
    return BlockConfig(hidden, heads, head_dim, ffn, default_sections(head_dim), **kw)


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# --- a1: timestep embedding and MLP ([card]: timestep layers in FP32) --------

def timestep_embedding(t: float, dim: int = 256, t_scale: float = 1000.0,
                       max_period: float = 10000.0) -> np.ndarray:
    """Sinusoidal embedding e(t) = [cos(t_scale t w_i) | sin(t_scale t w_i)],
    w_i = max_period^(-i/(dim/2)), i < dim/2."""
    half = dim // 2
    i = np.arange(half, dtype=np.float64)
    w = max_period ** (-i / half)
    arg = t_scale * float(t) * w
    return np.concatenate([np.cos(arg), np.sin(arg)])


def silu(x) -> np.ndarray:
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


def gelu(x, tanh: bool = False) -> np.ndarray:
    """GELU ([apx] "Activation Function: GELU"): x * Phi(x), exact erf form;
    the tanh approximation only when asked."""
    x = _f64(x)
    if tanh:
        return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def time_mlp(e, w_t1, b_t1, w_t2, b_t2) -> np.ndarray:
    """c = W_t2 SiLU(W_t1 e + b_t1) + b_t2 (weights in nn.Linear layout [out, in])."""
    h = silu(_f64(w_t1) @ _f64(e) + _f64(b_t1))
    return _f64(w_t2) @ h + _f64(b_t2)


def timestep_condition(t: float, tw: Dict[str, np.ndarray], cfg: BlockConfig) -> np.ndarray:
    e = timestep_embedding(t, cfg.time_dim, cfg.t_scale)
    return time_mlp(e, tw["w_t1"], tw["b_t1"], tw["w_t2"], tw["b_t2"])


# --- a2: AdaLN projection, once per step ([vllm] "AdaLN caching") -------------

def adaln_modulation(c, w_ada, b_ada) -> np.ndarray:
    """mod = W_ada SiLU(c) + b_ada, returned as [6, D]:
    shift1, scale1, gate1, shift2, scale2, gate2."""
    m = _f64(w_ada) @ silu(c) + _f64(b_ada)
    return m.reshape(6, -1)


# --- a3 / a7: RMSNorm then timestep scale/shift ([apx] diagram) ---------------

def rms_norm(x, eps: float) -> np.ndarray:
    """x / sqrt(mean_j x_j^2 + eps), per row, no learnable gain."""
    x = _f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def modulate(xn, shift, scale) -> np.ndarray:
    return _f64(xn) * (1.0 + _f64(scale)) + _f64(shift)


def norm_modulate(x, shift, scale, eps: float) -> np.ndarray:
    return modulate(rms_norm(x, eps), shift, scale)


# --- RoPE on the packed grid ([card] "3D multimodal RoPE") --------------------

def token_positions(n_txt: int, grids: Sequence[Tuple[int, int, int]]) -> np.ndarray:
    """(frame, row, col) of each token of the packed sequence
    [text; image 0; image 1; ...]. Text tokens sit at (0, 0, 0); image k's
    tokens are row-major over its (height, width) grid at its frame."""
    rows = [np.zeros((n_txt, 3), np.int64)]
    for frame, h, w in grids:
        r, c = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
        p = np.stack([np.full(h * w, frame), r.reshape(-1), c.reshape(-1)], axis=1)
        rows.append(p.astype(np.int64))
    return np.concatenate(rows, axis=0)


def rope_angles(pos: np.ndarray, sections: Sequence[int], theta: float) -> np.ndarray:
    """Angle of every rotation pair, [N, sum(sections)]: for axis a with s_a
    pairs, pair j turns by pos[:, a] * theta^(-j / s_a)."""
    out = []
    for a, s in enumerate(sections):
        j = np.arange(s, dtype=np.float64)
        w = theta ** (-j / s)
        out.append(_f64(pos[:, a])[:, None] * w[None, :])
    return np.concatenate(out, axis=1)


def apply_rope(x, pos: np.ndarray, sections: Sequence[int], theta: float) -> np.ndarray:
    """Rotate x [N, H, d] per head. Axis a owns channels [o_a, o_a + 2 s_a);
    pair j of that axis is (o_a + j, o_a + s_a + j) and turns by its angle:
    (x1, x2) -> (x1 cos - x2 sin, x2 cos + x1 sin)."""
    x = _f64(x)
    d = x.shape[-1]
    if 2 * sum(sections) != d:
        raise ValueError("rope sections do not cover head_dim")
    ang = rope_angles(pos, sections, theta)
    out = x.copy()
    o = 0
    p = 0
    for s in sections:
        cos = np.cos(ang[:, p:p + s])[:, None, :]
        sin = np.sin(ang[:, p:p + s])[:, None, :]
        x1 = x[..., o:o + s]
        x2 = x[..., o + s:o + 2 * s]
        out[..., o:o + s] = x1 * cos - x2 * sin
        out[..., o + s:o + 2 * s] = x2 * cos + x1 * sin
        o += 2 * s
        p += s
    return out


# --- a5: joint bidirectional attention ([card] single stream, [apx] 56/56 heads)

def attention(q, k, v) -> np.ndarray:
    """Per head h: O_h = softmax(Q_h K_h^T / sqrt(d)) V_h over all keys, no mask.
    q [R, H, d], k and v [N, H, d] -> [R, H, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    d = q.shape[-1]
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) / math.sqrt(d)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out


# --- a4 .. a9: the block ------------------------------------------------------

def linear(x, w) -> np.ndarray:
    """x W^T for an nn.Linear weight [out, in], no bias."""
    return _f64(x) @ _f64(w).T


def qkv_rope(xm, w_qkv, pos, cfg: BlockConfig):
    """Q, K, V [N, H, d] from the modulated tokens; RoPE on Q and K."""
    n = xm.shape[0]
    I = cfg.inner
    y = linear(xm, w_qkv)
    q = y[:, :I].reshape(n, cfg.heads, cfg.head_dim)
    k = y[:, I:2 * I].reshape(n, cfg.heads, cfg.head_dim)
    v = y[:, 2 * I:].reshape(n, cfg.heads, cfg.head_dim)
    q = apply_rope(q, pos, cfg.rope_sections, cfg.rope_theta)
    k = apply_rope(k, pos, cfg.rope_sections, cfg.rope_theta)
    return q, k, v


def block_forward(x, mod, w: Dict[str, np.ndarray], pos: np.ndarray, cfg: BlockConfig,
                  rows: Optional[Iterable[int]] = None) -> np.ndarray:
    """One DiT block on the packed sequence x [N, D] ([apx] diagram order):

        xm = RMSNorm(x) (1 + scale1) + shift1
        Q, K, V = xm W_q^T, xm W_k^T, xm W_v^T;  Q, K <- RoPE(pos)
        x  = x + gate1 * (Attention(Q, K, V) W_o^T)
        hm = RMSNorm(x) (1 + scale2) + shift2
        y  = x + gate2 * (GELU(hm W_1^T) W_2^T)

    With `rows`, only those output rows are computed (K and V still over all
    tokens, since every token attends to all of them); everything outside the
    attention is row-wise, so this equals selecting the rows of the full result.
    """
    x = _f64(x)
    n = x.shape[0]
    sh1, sc1, g1, sh2, sc2, g2 = _f64(mod)
    idx = np.arange(n) if rows is None else np.asarray(list(rows), dtype=np.int64)
    I = cfg.inner
    H, d = cfg.heads, cfg.head_dim
    wq = _f64(w["w_qkv"])[:I]
    wk = _f64(w["w_qkv"])[I:2 * I]
    wv = _f64(w["w_qkv"])[2 * I:]

    xm = norm_modulate(x, sh1, sc1, cfg.norm_eps)
    k = apply_rope(linear(xm, wk).reshape(n, H, d), pos, cfg.rope_sections, cfg.rope_theta)
    v = linear(xm, wv).reshape(n, H, d)
    q = apply_rope(linear(xm[idx], wq).reshape(len(idx), H, d), pos[idx],
                   cfg.rope_sections, cfg.rope_theta)
    o = attention(q, k, v).reshape(len(idx), I)

    xr = x[idx] + g1 * linear(o, w["w_o"])
    hm = norm_modulate(xr, sh2, sc2, cfg.norm_eps)
    u = gelu(linear(hm, w["w_ff1"]), cfg.gelu_tanh)
    return xr + g2 * linear(u, w["w_ff2"])


def pack(x_txt, x_img) -> np.ndarray:
    """The single-stream sequence [text; image tokens] ([card])."""
    return np.concatenate([_f64(x_txt), _f64(x_img)], axis=0)


def step_forward(x, t: float, tw: Dict[str, np.ndarray], blocks: Sequence[Dict[str, np.ndarray]],
                 pos: np.ndarray, cfg: BlockConfig) -> np.ndarray:
    """One denoising step: the timestep condition and every block's AdaLN
    modulation once ([vllm] "AdaLN caching"), then the blocks in order."""
    c = timestep_condition(t, tw, cfg)
    x = _f64(x)
    for w in blocks:
        mod = adaln_modulation(c, w["w_ada"], w["b_ada"])
        x = block_forward(x, mod, w, pos, cfg)
    return x


# --- a11: MXFP8 block-scaled linears ("H3-Image Day-0 Support", "Faster DiT":
# MXFP8 GEMMs for the eligible DiT linears) ------------------------------------
# The pages name the format only. Reading: the OCP Microscaling (MX) v1.0
# format - E4M3 elements (bias 7, 3 mantissa bits, no infinities, largest
# finite 448) sharing one E8M0 scale 2^X per 32 consecutive elements along
# the reduction axis, X = floor(log2(amax)) - 8 (8 = exponent of E4M3's
# largest normal); elements rounded to nearest, ties to even, saturating at
# +-448. All four block linears (QKV, out-projection, FFN1, FFN2) are
# eligible, for both operands; attention stays bf16.

MX_BLOCK = 32
E4M3_MAX = 448.0


def e4m3_round(v) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even), saturating at +-448.
    Normal values 2^e (1 + m/8), e in [-6, 8]; subnormals m/8 * 2^-6."""
    v = _f64(v)
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)
    quantum = 2.0 ** (e - 3)
    q = np.round(a / quantum) * quantum  # numpy rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.sign(v) * q


def mx_scale_exponent(amax) -> np.ndarray:
    """X = floor(log2(amax)) - 8 per block; blocks of zeros get the smallest
    E8M0 exponent, -127."""
    amax = _f64(amax)
    with np.errstate(divide="ignore"):
        x = np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 8
    return np.where(amax > 0, np.clip(x, -127, 127), -127.0)


def mx_quantize(x):
    """MXFP8 along the last axis (length a multiple of 32): returns the E4M3
    element values and the per-block scale exponents X (value = q * 2^X)."""
    x = _f64(x)
    k = x.shape[-1]
    if k % MX_BLOCK:
        raise ValueError("last axis must be a multiple of 32")
    blocks = x.reshape(x.shape[:-1] + (k // MX_BLOCK, MX_BLOCK))
    X = mx_scale_exponent(np.max(np.abs(blocks), axis=-1))
    q = e4m3_round(blocks / 2.0 ** X[..., None])
    return q.reshape(x.shape), X


def mx_dequantize(q, X) -> np.ndarray:
    q = _f64(q)
    k = q.shape[-1]
    blocks = q.reshape(q.shape[:-1] + (k // MX_BLOCK, MX_BLOCK))
    return (blocks * 2.0 ** _f64(X)[..., None]).reshape(q.shape)


def mx_roundtrip(x) -> np.ndarray:
    return mx_dequantize(*mx_quantize(x))


def linear_mx(x, w) -> np.ndarray:
    """x W^T with both operands MXFP8-quantized along the reduction axis."""
    return mx_roundtrip(x) @ mx_roundtrip(w).T


def block_forward_mx(x, mod, w: Dict[str, np.ndarray], pos: np.ndarray, cfg: BlockConfig,
                     rows: Optional[Iterable[int]] = None) -> np.ndarray:
    """block_forward with the four linears on MXFP8 operands (a11)."""
    x = _f64(x)
    n = x.shape[0]
    sh1, sc1, g1, sh2, sc2, g2 = _f64(mod)
    idx = np.arange(n) if rows is None else np.asarray(list(rows), dtype=np.int64)
    I = cfg.inner
    H, d = cfg.heads, cfg.head_dim
    wqkv = mx_roundtrip(w["w_qkv"])
    xm = mx_roundtrip(norm_modulate(x, sh1, sc1, cfg.norm_eps))
    k = apply_rope((xm @ wqkv[I:2 * I].T).reshape(n, H, d), pos, cfg.rope_sections, cfg.rope_theta)
    v = (xm @ wqkv[2 * I:].T).reshape(n, H, d)
    q = apply_rope((xm[idx] @ wqkv[:I].T).reshape(len(idx), H, d), pos[idx],
                   cfg.rope_sections, cfg.rope_theta)
    o = attention(q, k, v).reshape(len(idx), I)
    xr = x[idx] + g1 * linear_mx(o, w["w_o"])
    hm = norm_modulate(xr, sh2, sc2, cfg.norm_eps)
    u = gelu(linear_mx(hm, w["w_ff1"]), cfg.gelu_tanh)
    return xr + g2 * linear_mx(u, w["w_ff2"])


# --- Around the block loop: patchify, embeddings, output layer, sampler ------
# [card] "Model Architecture": the image VAE has 16x spatial downsampling and
# 24 latent channels; the DiT patchifies the latent with a 2x2 patch (so one
# token covers 32x32 pixels); the embedding, timestep and output layers are
# FP32. The real per-step output heads and the sampling schedule ship in a
# file these pages do not give, so the plain reading stands in for them: a
# DiT final layer (RMSNorm, AdaLN shift/scale from the timestep condition,
# Linear D -> 96 with bias) predicting the flow velocity dz/dt, and Euler
# steps from t = 1 (noise) to t = 0 over the step_forward schedule.

LATENT_CHANNELS = 24
PATCH = 2


def patchify(z, patch: int = PATCH) -> np.ndarray:
    """Latent z [C, Hl, Wl] -> tokens [(Hl/p) (Wl/p), C p p]. Token (r, c) is
    row-major over the (Hl/p, Wl/p) grid, the order token_positions gives an
    image; feature ch * p^2 + i * p + j holds latent pixel (p r + i, p c + j)
    of channel ch."""
    z = _f64(z)
    C, Hl, Wl = z.shape
    if Hl % patch or Wl % patch:
        raise ValueError("latent sides must be multiples of the patch")
    h, w = Hl // patch, Wl // patch
    t = z.reshape(C, h, patch, w, patch)          # ch, r, i, c, j
    return t.transpose(1, 3, 0, 2, 4).reshape(h * w, C * patch * patch)


def unpatchify(tokens, channels: int, h: int, w: int, patch: int = PATCH) -> np.ndarray:
    """The inverse of patchify: tokens [h w, C p p] -> latent [C, h p, w p]."""
    t = _f64(tokens).reshape(h, w, channels, patch, patch)   # r, c, ch, i, j
    return t.transpose(2, 0, 3, 1, 4).reshape(channels, h * patch, w * patch)


def patch_embed(tokens, w, b) -> np.ndarray:
    """FP32 patch embedding ([card]): tokens [n, C p p] W^T + b -> [n, D]."""
    return _f64(tokens) @ _f64(w).T + _f64(b)


def final_layer(x, c, w_mod, b_mod, w_out, b_out, eps: float) -> np.ndarray:
    """Output layer on the image tokens x [n, D]: [shift, scale] =
    W_mod SiLU(c) + b_mod (W_mod [2D, D]), then
    (RMSNorm(x) (1 + scale) + shift) W_out^T + b_out (W_out [C p p, D])."""
    shift, scale = (_f64(w_mod) @ silu(c) + _f64(b_mod)).reshape(2, -1)
    return norm_modulate(x, shift, scale, eps) @ _f64(w_out).T + _f64(b_out)


def sampling_timesteps(n_steps: int) -> np.ndarray:
    """t_k = 1 - k / n for k = 0 .. n: the n network evaluations happen at
    t_0 .. t_{n-1}, and the last Euler step lands on t_n = 0."""
    return 1.0 - np.arange(n_steps + 1, dtype=np.float64) / n_steps


def euler_update(z, v, t: float, t_next: float) -> np.ndarray:
    """One step of dz/dt = v: z(t_next) = z(t) + (t_next - t) v."""
    return _f64(z) + (float(t_next) - float(t)) * _f64(v)


def dit_velocity(z, x_txt, t: float, tw: Dict[str, np.ndarray],
                 blocks: Sequence[Dict[str, np.ndarray]], io: Dict[str, np.ndarray],
                 cfg: BlockConfig) -> np.ndarray:
    """The denoiser on one target latent z [C, Hl, Wl] with text tokens
    x_txt [n_txt, D]: patchify, embed, the packed step through every block,
    the output layer on the image tokens, unpatchify. io holds w_in [D, 96],
    b_in [D], w_mod [2D, D], b_mod [2D], w_out [96, D], b_out [96]."""
    C, Hl, Wl = _f64(z).shape
    h, w = Hl // PATCH, Wl // PATCH
    x_img = patch_embed(patchify(z), io["w_in"], io["b_in"])
    n_txt = _f64(x_txt).shape[0]
    pos = token_positions(n_txt, [(0, h, w)])
    y = step_forward(pack(x_txt, x_img), t, tw, blocks, pos, cfg)
    c = timestep_condition(t, tw, cfg)
    out = final_layer(y[n_txt:], c, io["w_mod"], io["b_mod"], io["w_out"], io["b_out"],
                      cfg.norm_eps)
    return unpatchify(out, C, h, w)


def denoise(z_noise, velocity, n_steps: int) -> np.ndarray:
    """Euler integration of dz/dt = velocity(z, t) from t = 1 to t = 0 over
    sampling_timesteps(n_steps); velocity is any callable (the DiT above, or a
    closed-form field in the tests)."""
    ts = sampling_timesteps(n_steps)
    z = _f64(z_noise)
    for k in range(n_steps):
        z = euler_update(z, velocity(z, ts[k]), ts[k], ts[k + 1])
    return z


def block_flops(n: int, hidden: int, inner: int, ffn: int) -> int:
    """Algorithmic flops of one block: QKV 6NDI, out-proj 2NDI, FFN 4NDF,
    attention 4N^2 I (QK^T and PV over all N^2 pairs, no causal halving)."""
    return 8 * n * hidden * inner + 4 * n * hidden * ffn + 4 * n * n * inner
