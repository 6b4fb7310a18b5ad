"""Pins for the oracle's steps around the block loop (patchify, the FP32
patch embedding and output layer, the Euler sampler), each against something
other than the oracle's own formula: brute-force index loops, torch layers,
exact inverses and a closed-form flow. CPU only."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from image_generation_b200 import synth
from oracle import dit_block as O


def test_patchify_layout_by_brute_force():
    """Every latent element lands where the stated layout puts it."""
    C, Hl, Wl, p = 3, 4, 6, 2
    z = np.random.default_rng(0).standard_normal((C, Hl, Wl))
    tok = O.patchify(z, p)
    w = Wl // p
    assert tok.shape == ((Hl // p) * w, C * p * p)
    for ch in range(C):
        for y in range(Hl):
            for x in range(Wl):
                r, i = divmod(y, p)
                c, j = divmod(x, p)
                assert tok[r * w + c, ch * p * p + i * p + j] == z[ch, y, x]


def test_patchify_matches_token_grid_and_inverts():
    """The token order is the grid order token_positions assigns an image, and
    unpatchify undoes patchify exactly (24 channels, 2x2 patches)."""
    Hl, Wl = 10, 14
    z = np.random.default_rng(1).standard_normal((O.LATENT_CHANNELS, Hl, Wl))
    tok = O.patchify(z)
    assert tok.shape == (Hl * Wl // 4, 96)
    pos = O.token_positions(0, [(0, Hl // 2, Wl // 2)])
    # the top-left latent pixel of each token's patch sits at 2 x its (row, col)
    for n in (0, 1, Wl // 2, tok.shape[0] - 1):
        _, r, c = pos[n]
        assert tok[n, 0] == z[0, 2 * r, 2 * c]
    assert np.array_equal(O.unpatchify(tok, O.LATENT_CHANNELS, Hl // 2, Wl // 2), z)


def test_patchify_equals_pixel_unshuffle():
    """torch's pixel_unshuffle groups a channel's p x p block the same way."""
    z = np.random.default_rng(2).standard_normal((O.LATENT_CHANNELS, 6, 8))
    ref = F.pixel_unshuffle(torch.from_numpy(z)[None], 2)[0]        # [C p p, h, w]
    ref = ref.permute(1, 2, 0).reshape(-1, O.LATENT_CHANNELS * 4).numpy()
    assert np.array_equal(O.patchify(z), ref)


def test_patch_embed_and_output_layer_against_torch():
    g = np.random.default_rng(3)
    D, n = 64, 9
    tok = g.standard_normal((n, 96))
    w_in, b_in = g.standard_normal((D, 96)) * 0.1, g.standard_normal(D)
    ref = F.linear(torch.from_numpy(tok), torch.from_numpy(w_in), torch.from_numpy(b_in)).numpy()
    np.testing.assert_allclose(O.patch_embed(tok, w_in, b_in), ref, rtol=1e-12, atol=1e-12)

    x = g.standard_normal((n, D)) * 3
    c = g.standard_normal(D)
    w_mod, b_mod = g.standard_normal((2 * D, D)) * 0.2, g.standard_normal(2 * D) * 0.2
    w_out, b_out = g.standard_normal((96, D)) * 0.1, g.standard_normal(96)
    tx = torch.from_numpy
    mod = F.linear(F.silu(tx(c)), tx(w_mod), tx(b_mod))
    shift, scale = mod[:D], mod[D:]
    h = F.rms_norm(tx(x), (D,), eps=1e-6) * (1 + scale) + shift
    ref = F.linear(h, tx(w_out), tx(b_out)).numpy()
    got = O.final_layer(x, c, w_mod, b_mod, w_out, b_out, 1e-6)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)
    # no modulation: plain RMSNorm then the linear
    plain = F.linear(F.rms_norm(tx(x), (D,), eps=1e-6), tx(w_out), tx(b_out)).numpy()
    zero = O.final_layer(x, c, np.zeros_like(w_mod), np.zeros(2 * D), w_out, b_out, 1e-6)
    np.testing.assert_allclose(zero, plain, rtol=1e-10, atol=1e-10)


def test_schedule_and_euler_on_a_straight_flow():
    """On the straight path z_t = t noise + (1 - t) x0 the velocity is the
    constant noise - x0, so Euler steps land on x0 for any step count."""
    ts = O.sampling_timesteps(6)
    assert ts[0] == 1.0 and ts[-1] == 0.0 and len(ts) == 7 and np.all(np.diff(ts) < 0)
    g = np.random.default_rng(4)
    x0, noise = g.standard_normal((24, 8, 8)), g.standard_normal((24, 8, 8))
    calls = []

    def v(z, t):
        calls.append(t)
        return noise - x0

    for n in (1, 6, 11):
        calls.clear()
        np.testing.assert_allclose(O.denoise(noise, v, n), x0, rtol=0, atol=1e-12)
        assert calls == list(O.sampling_timesteps(n)[:-1])
    # a field linear in z: dz/dt = -z from t = 1 gives z(0) = z(1) e, and
    # Euler with n steps gives z(1) (1 + 1/n)^n
    z1 = g.standard_normal(5)
    for n in (1, 6, 50):
        np.testing.assert_allclose(O.denoise(z1, lambda z, t: -z, n), z1 * (1 + 1 / n) ** n, rtol=1e-12)


def _io_weights(D, seed):
    g = np.random.default_rng(seed)
    return {"w_in": g.standard_normal((D, 96)) * 0.05, "b_in": g.standard_normal(D) * 0.1,
            "w_mod": g.standard_normal((2 * D, D)) * 0.02, "b_mod": g.standard_normal(2 * D) * 0.1,
            "w_out": g.standard_normal((96, D)) * 0.05, "b_out": g.standard_normal(96) * 0.1}


def test_velocity_with_identity_blocks_is_embed_then_output_layer():
    """Zero gates make every block the identity, so the denoiser reduces to
    unpatchify(output layer(patch embedding(patchify(z)))), text unused."""
    d = synth.Dims(64, 2, 96, 128)
    cfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
    tw = synth.time_weights(d, 5)
    blocks = []
    for l in range(2):
        bw = synth.block_weights(d, 10 + l)
        bw["w_ada"][2 * d.hidden:3 * d.hidden] = 0
        bw["w_ada"][5 * d.hidden:] = 0
        blocks.append(bw)
    io = _io_weights(d.hidden, 6)
    z = np.random.default_rng(7).standard_normal((24, 4, 6))
    t = 0.7
    c = O.timestep_condition(t, tw, cfg)
    expect = O.unpatchify(O.final_layer(O.patch_embed(O.patchify(z), io["w_in"], io["b_in"]), c,
                                        io["w_mod"], io["b_mod"], io["w_out"], io["b_out"],
                                        cfg.norm_eps), 24, 2, 3)
    for x_txt in (synth.tokens(3, d.hidden, 8, "t"), synth.tokens(5, d.hidden, 9, "t")):
        v = O.dit_velocity(z, x_txt, t, tw, blocks, io, cfg)
        assert v.shape == z.shape
        np.testing.assert_allclose(v, expect, rtol=1e-12, atol=1e-12)


def test_velocity_reads_the_text_through_attention():
    """With live gates the image velocity depends on the text tokens."""
    d = synth.Dims(64, 2, 96, 128)
    cfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
    tw = synth.time_weights(d, 5)
    blocks = [synth.block_weights(d, 20)]
    blocks[0]["w_ada"] = synth.normal_bf16((6 * d.hidden, d.hidden), 0.5, 21, "w_ada")
    io = _io_weights(d.hidden, 6)
    z = np.random.default_rng(7).standard_normal((24, 4, 4))
    v1 = O.dit_velocity(z, synth.tokens(3, d.hidden, 8, "t"), 0.4, tw, blocks, io, cfg)
    v2 = O.dit_velocity(z, synth.tokens(3, d.hidden, 9, "t"), 0.4, tw, blocks, io, cfg)
    assert np.abs(v1 - v2).max() > 1e-6


@pytest.mark.parametrize("shape", [(24, 3, 4), (24, 4, 5)])
def test_patchify_rejects_odd_sides(shape):
    with pytest.raises(ValueError):
        O.patchify(np.zeros(shape))
