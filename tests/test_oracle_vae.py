"""Pins for the VAE decoder oracle (oracle/vae_decoder.py), each against
something other than the oracle's own formula: torch's LayerNorm and its
pre-norm TransformerEncoderLayer (GELU, biases) loaded with the same weights,
torch's pixel_shuffle and brute-force index loops, closed forms of the
position table, the tiling's partition and independence properties, and a
count of products for the flop formula. CPU only."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from image_generation_b200 import synth
from oracle import vae_decoder as V

CFG = V.VaeConfig(width=64, heads=4, head_dim=16, mlp=256, layers=2, tile=4)


def _weights(cfg, seed=0):
    v = synth.VaeDims(width=cfg.width, heads=cfg.heads, head_dim=cfg.head_dim, mlp=cfg.mlp,
                      layers=cfg.layers, tile=cfg.tile)
    return synth.vae_weights(v, seed, std=0.1)


def test_layer_norm_against_torch():
    g = np.random.default_rng(0)
    x = g.standard_normal((7, 64)) * 3 + 1.5
    gain, bias = g.standard_normal(64), g.standard_normal(64)
    ref = F.layer_norm(torch.from_numpy(x), (64,), torch.from_numpy(gain), torch.from_numpy(bias),
                       eps=1e-6).numpy()
    np.testing.assert_allclose(V.layer_norm(x, gain, bias, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_vit_layer_against_torch_encoder_layer():
    """A pre-norm torch.nn.TransformerEncoderLayer (exact GELU, biases, eps
    1e-6) holding the same weights computes the same layer."""
    w = _weights(CFG)["layers"][0]
    W = CFG.width
    layer = torch.nn.TransformerEncoderLayer(W, CFG.heads, CFG.mlp, dropout=0.0, activation="gelu",
                                             layer_norm_eps=CFG.eps, batch_first=True,
                                             norm_first=True).double().eval()
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(t(w["w_qkv"]))
        layer.self_attn.in_proj_bias.copy_(t(w["b_qkv"]))
        layer.self_attn.out_proj.weight.copy_(t(w["w_o"]))
        layer.self_attn.out_proj.bias.copy_(t(w["b_o"]))
        layer.linear1.weight.copy_(t(w["w_1"]))
        layer.linear1.bias.copy_(t(w["b_1"]))
        layer.linear2.weight.copy_(t(w["w_2"]))
        layer.linear2.bias.copy_(t(w["b_2"]))
        layer.norm1.weight.copy_(t(w["ln1_g"]))
        layer.norm1.bias.copy_(t(w["ln1_b"]))
        layer.norm2.weight.copy_(t(w["ln2_g"]))
        layer.norm2.bias.copy_(t(w["ln2_b"]))
        x = np.random.default_rng(1).standard_normal((12, W))
        ref = layer(t(x)[None])[0].numpy()
    np.testing.assert_allclose(V.vit_layer(x, w, CFG), ref, rtol=1e-10, atol=1e-10)


def test_position_table_closed_forms():
    h, w, W = 3, 5, 64
    pe = V.position_table(h, w, W)
    q = W // 4
    assert pe.shape == (h * w, W)
    # position (0, 0): sin 0 = 0, cos 0 = 1 in both halves
    assert np.array_equal(pe[0], np.concatenate([np.zeros(q), np.ones(q), np.zeros(q), np.ones(q)]))
    # frequency 1 channels (k = 0) hold sin r, cos r, sin c, cos c
    for n in range(h * w):
        r, c = divmod(n, w)
        assert pe[n, 0] == math.sin(r) and pe[n, q] == math.cos(r)
        assert pe[n, 2 * q] == math.sin(c) and pe[n, 3 * q] == math.cos(c)
    # the last frequency is 10000^(-(q-1)/q)
    assert np.isclose(pe[w + 1, q - 1], math.sin(10000.0 ** (-(q - 1) / q)), rtol=1e-15)
    # each half's inner products depend only on the offset (rotations)
    rows = V.position_table(9, 1, W)[:, :W // 2]
    assert np.isclose(rows[2] @ rows[5], rows[4] @ rows[7], rtol=1e-12)


def test_unpatchify_pixels_by_brute_force_and_pixel_shuffle():
    h, w = 2, 3
    y = np.random.default_rng(2).standard_normal((h * w, 768))
    img = V.unpatchify_pixels(y, h, w)
    assert img.shape == (3, 32, 48)
    for r in range(h):
        for c in range(w):
            for ch in range(3):
                for i in range(16):
                    for j in range(16):
                        assert img[ch, 16 * r + i, 16 * c + j] == y[r * w + c, ch * 256 + 16 * i + j]
    ref = F.pixel_shuffle(torch.from_numpy(y.T.reshape(768, h, w))[None], 16)[0].numpy()
    assert np.array_equal(img, ref)


@pytest.mark.parametrize("shape", [(8, 8), (9, 6), (3, 10)])
def test_tiles_partition_the_latent(shape):
    h, w = shape
    cover = np.zeros(shape, np.int64)
    for r0, c0, th, tw in V.tiles(h, w, 4):
        assert 1 <= th <= 4 and 1 <= tw <= 4 and r0 % 4 == 0 and c0 % 4 == 0
        cover[r0:r0 + th, c0:c0 + tw] += 1
    assert np.all(cover == 1)


def test_decode_is_tile_local_and_independent():
    """One tile decodes the same wherever it sits (the table is tile-local);
    changing one tile's latent changes only that tile's pixels; a ragged
    latent decodes its edge tiles at their own sizes."""
    weights = _weights(CFG)
    g = np.random.default_rng(3)
    z = g.standard_normal((24, 8, 7))
    img = V.decode(z, weights, CFG)
    assert img.shape == (3, 128, 112)
    tile = V.decode_tile(z[:, 4:8, 4:7], weights, CFG)
    assert np.array_equal(img[:, 64:128, 64:112], tile)
    z2 = z.copy()
    z2[:, 0:4, 4:7] += g.standard_normal((24, 4, 3))
    img2 = V.decode(z2, weights, CFG)
    changed = np.abs(img2 - img) > 0
    assert changed[:, 0:64, 64:112].any()
    changed[:, 0:64, 64:112] = False
    assert not changed.any()
    # the same latent block decoded at another tile position
    z3 = np.concatenate([z[:, 0:4, 0:4], z[:, 0:4, 0:4]], axis=2)
    img3 = V.decode(z3, weights, CFG)
    assert np.array_equal(img3[:, :, :64], img3[:, :, 64:])


def test_decode_tile_against_a_torch_encoder_stack():
    """The whole tile: embedding + table, the layers as torch encoder layers,
    final LayerNorm and output linear, pixel_shuffle to pixels."""
    weights = _weights(CFG, seed=4)
    z = np.random.default_rng(4).standard_normal((24, 4, 3))
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    x = t(z.reshape(24, 12).T) @ t(weights["w_in"]).T + t(weights["b_in"])
    x = x + t(V.position_table(4, 3, CFG.width))
    for w in weights["layers"]:
        layer = torch.nn.TransformerEncoderLayer(CFG.width, CFG.heads, CFG.mlp, dropout=0.0,
                                                 activation="gelu", layer_norm_eps=CFG.eps,
                                                 batch_first=True, norm_first=True).double().eval()
        sd = {"self_attn.in_proj_weight": w["w_qkv"], "self_attn.in_proj_bias": w["b_qkv"],
              "self_attn.out_proj.weight": w["w_o"], "self_attn.out_proj.bias": w["b_o"],
              "linear1.weight": w["w_1"], "linear1.bias": w["b_1"], "linear2.weight": w["w_2"],
              "linear2.bias": w["b_2"], "norm1.weight": w["ln1_g"], "norm1.bias": w["ln1_b"],
              "norm2.weight": w["ln2_g"], "norm2.bias": w["ln2_b"]}
        layer.load_state_dict({k: t(v) for k, v in sd.items()})
        with torch.no_grad():
            x = layer(x[None])[0]
    y = F.layer_norm(x, (CFG.width,), t(weights["lnf_g"]), t(weights["lnf_b"]), eps=CFG.eps)
    y = y @ t(weights["w_out"]).T + t(weights["b_out"])
    ref = F.pixel_shuffle(y.T.reshape(768, 4, 3)[None], 16)[0].detach().numpy()
    np.testing.assert_allclose(V.decode_tile(z, weights, CFG), ref, rtol=1e-9, atol=1e-9)


def test_decode_flops_against_a_count_of_products():
    cfg = V.VaeConfig(width=8, heads=2, head_dim=4, mlp=32, layers=3, tile=4)
    Hl, Wl = 6, 5
    count = 0
    for _, _, h, w in V.tiles(Hl, Wl, cfg.tile):
        n = h * w
        count += n * cfg.channels * cfg.width                      # embedding
        per_layer = n * cfg.width * 3 * cfg.width + n * cfg.width * cfg.width \
            + n * cfg.width * cfg.mlp * 2                           # qkv, o, mlp
        per_layer += 2 * n * n * cfg.width                          # QK^T and PV
        count += cfg.layers * per_layer
        count += n * cfg.width * cfg.out_features                  # output linear
    assert V.decode_flops(Hl, Wl, cfg) == 2 * count


def test_vae_shapes_follow_the_pages():
    """24 layers, 24 latent channels, 16x per side; the reading's widths give
    about 0.47B decoder parameters (the pages' VAE is 0.58B with its encoder)."""
    cfg = V.VaeConfig()
    assert cfg.layers == 24 and cfg.channels == 24 and V.SCALE == 16
    W, M = cfg.width, cfg.mlp
    per_layer = 3 * W * W + 3 * W + W * W + W + W * M + M + M * W + W + 4 * W
    params = cfg.layers * per_layer + 24 * W + W + 2 * W + 768 * W + 768
    assert 0.45e9 < params < 0.58e9
