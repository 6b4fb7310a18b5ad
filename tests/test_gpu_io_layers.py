"""GPU parity of the steps around the block loop (patchify + FP32 patch
embedding, the output layer's modulation, output layer + unpatchify + Euler
step) against the oracle, and a short denoise loop through all of them."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import (assert_bf16_rounding, assert_close, block_tensors, time_tensors,
                           to_dev, to_np)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ctx(dims, n_blocks=1, max_tokens=512, io_fp32=False, seed=0):
    from image_generation_b200 import h3dit as H

    tw = synth.time_weights(dims, seed)
    bws = [synth.block_weights(dims, seed + 1000 + l) for l in range(n_blocks)]
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, max_tokens,
                        io_fp32=io_fp32)
    return H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws]), tw, bws


def _io(D, C, seed):
    f = lambda shape, std, tag: synth.normal_f32(shape, std, seed, tag)
    return {"w_in": f((D, 4 * C), 0.05, "w_in"), "b_in": f((D,), 0.1, "b_in"),
            "w_mod": f((2 * D, D), 0.02, "w_mod"), "b_mod": f((2 * D,), 0.1, "b_mod"),
            "w_out": f((4 * C, D), 0.05, "w_out"), "b_out": f((4 * C,), 0.1, "b_out")}


@pytest.mark.parametrize("io_fp32", [False, True], ids=["bf16_tokens", "fp32_tokens"])
@pytest.mark.parametrize("shape", [(24, 32, 32), (24, 18, 26), (3, 4, 6)],
                         ids=["24x32x32", "ragged_24x18x26", "3ch_4x6"])
def test_embed_latent(shape, io_fp32):
    dims = synth.SMALL
    ctx, _, _ = _ctx(dims, io_fp32=io_fp32)
    C, Hl, Wl = shape
    z = synth.normal_f32(shape, 1.0, 1, "z")
    io = _io(dims.hidden, C, 2)
    n = (Hl // 2) * (Wl // 2)
    out = torch.full((n, dims.hidden), float("nan"), device="cuda",
                     dtype=torch.float32 if io_fp32 else torch.bfloat16)
    ctx.embed_latent(to_dev(z, "f32"), to_dev(io["w_in"], "f32"), to_dev(io["b_in"], "f32"), out)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    ref = O.patch_embed(O.patchify(z), io["w_in"], io["b_in"])
    got = to_np(out)
    if io_fp32:
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    else:
        assert_bf16_rounding(got, ref, "patch embedding (bf16 tokens)")


def test_output_modulation():
    dims = synth.SMALL
    ctx, _, _ = _ctx(dims)
    D = dims.hidden
    io = _io(D, 24, 3)
    c = synth.normal_f32((D,), 1.0, 3, "c")
    mod = torch.empty(2 * D, device="cuda")
    ctx.output_modulation(to_dev(c, "f32"), to_dev(io["w_mod"], "f32"), to_dev(io["b_mod"], "f32"),
                          mod)
    torch.cuda.synchronize()
    ref = io["w_mod"].astype(np.float64) @ O.silu(c) + io["b_mod"]
    assert np.abs(to_np(mod) - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("io_fp32", [False, True], ids=["bf16_tokens", "fp32_tokens"])
@pytest.mark.parametrize("shape", [(24, 32, 32), (24, 18, 26)], ids=["24x32x32", "ragged_24x18x26"])
def test_output_euler(shape, io_fp32):
    dims = synth.SMALL
    D = dims.hidden
    ctx, _, _ = _ctx(dims, io_fp32=io_fp32)
    C, Hl, Wl = shape
    n = (Hl // 2) * (Wl // 2)
    x = synth.tokens(n, D, 4, "x")  # bf16-representable, so both token dtypes carry it exactly
    mod = synth.normal_f32((2, D), 0.2, 4, "mod")
    io = _io(D, C, 4)
    z = synth.normal_f32(shape, 1.0, 4, "z")
    dt = -1.0 / 6.0
    zd = to_dev(z, "f32")
    ctx.output_euler(to_dev(x, "f32" if io_fp32 else "bf16"), to_dev(mod.reshape(-1), "f32"),
                     to_dev(io["w_out"], "f32"), to_dev(io["b_out"], "f32"), zd, dt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    v = O.unpatchify(O.norm_modulate(x, mod[0], mod[1], 1e-6) @ io["w_out"].T.astype(np.float64)
                     + io["b_out"], C, Hl // 2, Wl // 2)
    got_v = (to_np(zd).astype(np.float64) - z) / dt
    assert_close(got_v, v, "output layer velocity", cos_min=0.999999, rel_max=1e-4)


def test_short_denoise_loop_matches_oracle():
    """Two Euler steps of the whole denoiser (patchify + embedding, one block
    through h3dit_step, output layer + Euler) on a 24 x 16 x 16 latent with 8
    text tokens, against the oracle's denoise with its velocity function."""
    dims = synth.SMALL
    D = dims.hidden
    ctx, tw, bws = _ctx(dims, io_fp32=True)
    C, Hl, Wl, n_txt = 24, 16, 16, 8
    h, w = Hl // 2, Wl // 2
    io = _io(D, C, 5)
    x_txt = synth.tokens(n_txt, D, 5, "txt")
    z0 = synth.normal_f32((C, Hl, Wl), 1.0, 5, "z")
    dev = {k: to_dev(v, "f32") for k, v in io.items()}
    zd = to_dev(z0, "f32")
    txt = torch.empty(n_txt, D, device="cuda")
    img = torch.empty(h * w, D, device="cuda")
    c = torch.empty(D, device="cuda")
    mod = torch.empty(2 * D, device="cuda")
    ts = O.sampling_timesteps(2)
    for k in range(2):
        t, t_next = float(ts[k]), float(ts[k + 1])
        txt.copy_(to_dev(x_txt, "f32"))          # the text states are the same every step
        ctx.embed_latent(zd, dev["w_in"], dev["b_in"], img)
        ctx.step(t, img, [(0, h, w)], txt)
        ctx.time_embed(t, c)
        ctx.output_modulation(c, dev["w_mod"], dev["b_mod"], mod)
        ctx.output_euler(img, mod, dev["w_out"], dev["b_out"], zd, t_next - t)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    cfg = O.config_for(D, dims.heads, dims.head_dim, dims.ffn)
    velocity = lambda z, t: O.dit_velocity(z, x_txt, t, tw, bws, io, cfg)
    ref = O.denoise(z0, velocity, 2)
    got = to_np(zd).astype(np.float64)
    assert_close(got - z0, ref - z0, "two-step denoise (latent change)", cos_min=0.9999)


def test_latent_shape_errors():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    ctx, _, _ = _ctx(dims, max_tokens=64)
    D = dims.hidden
    w_in = torch.zeros(D, 96, device="cuda")
    b_in = torch.zeros(D, device="cuda")
    out = torch.zeros(256, D, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(H.H3DitError) as e:   # odd side
        ctx.embed_latent(torch.zeros(24, 5, 4, device="cuda"), w_in, b_in, out)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    with pytest.raises(H.H3DitError) as e:   # more tokens than max_tokens
        ctx.embed_latent(torch.zeros(24, 32, 32, device="cuda"), w_in, b_in, out)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    with pytest.raises(H.H3DitError) as e:   # too many channels
        ctx.embed_latent(torch.zeros(40, 4, 4, device="cuda"), torch.zeros(D, 160, device="cuda"),
                         b_in, out)
    assert e.value.status == H.H3DIT_ERR_UNSUPPORTED
    assert ctx.sync_status() == 0


_DENOISE_REF = {}


def _denoise_case(n_blocks, gate_bias):
    """Weights and inputs of the whole-loop test: width 768 (the small
    workload's widths), a 24 x 32 x 32 latent (a 16 x 16 patch grid, 256 image
    tokens) and 32 text tokens - the small workload's 288 tokens, so the
    linears run on the paired-CTA kernel. gate_bias is added to both gate
    chunks of every b_ada, so that the blocks' branches reach the output at
    full strength instead of the ~2% of the N(0, 0.02) init."""
    dims = synth.SMALL
    D = dims.hidden
    tw = synth.time_weights(dims, 11)
    bws = []
    for l in range(n_blocks):
        b = synth.block_weights(dims, 1100 + l)
        b["b_ada"] = b["b_ada"].copy()
        b["b_ada"][2 * D:3 * D] += gate_bias
        b["b_ada"][5 * D:6 * D] += gate_bias
        bws.append(b)
    io = _io(D, 24, 12)
    x_txt = synth.tokens(32, D, 13, "txt")
    z0 = synth.normal_f32((24, 32, 32), 1.0, 13, "z")
    return dims, tw, bws, io, x_txt, z0


def _denoise_reference(n_blocks, gate_bias, n_steps):
    key = (n_blocks, gate_bias, n_steps)
    if key not in _DENOISE_REF:
        dims, tw, bws, io, x_txt, z0 = _denoise_case(n_blocks, gate_bias)
        cfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
        velocity = lambda z, t: O.dit_velocity(z, x_txt, t, tw, bws, io, cfg)
        _DENOISE_REF[key] = O.denoise(z0, velocity, n_steps)
    return _DENOISE_REF[key]


@pytest.mark.parametrize("io_fp32", [False, True], ids=["bf16_tokens", "fp32_tokens"])
@pytest.mark.parametrize("n_blocks,gate_bias", [(50, 0.0), (3, 1.0)],
                         ids=["50_blocks", "3_blocks_full_gates"])
def test_denoise_matches_oracle(n_blocks, gate_bias, io_fp32):
    """h3dit_denoise: the whole 6-step sampling loop (timestep MLP, AdaLN
    projections, patch embedding, the blocks, output layer, Euler update) in
    one call, against the oracle's denoise over dit_velocity. The output is
    the denoised latent; its change from the noise is checked too, since the
    noise dominates it."""
    from image_generation_b200 import h3dit as H

    n_steps = synth.N_STEPS
    dims, tw, bws, io, x_txt, z0 = _denoise_case(n_blocks, gate_bias)
    D = dims.hidden
    cfg = H.make_config(D, dims.heads, dims.head_dim, dims.ffn, n_blocks, 288, io_fp32=io_fp32)
    ctx = H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws])
    zd = to_dev(z0, "f32")
    txt = to_dev(x_txt, "f32" if io_fp32 else "bf16")
    txt0 = txt.clone()
    ctx.denoise({k: to_dev(v, "f32") for k, v in io.items()}, zd, txt, n_steps)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    assert torch.equal(txt, txt0), "the text states are read only"
    ref = _denoise_reference(n_blocks, gate_bias, n_steps)
    got = to_np(zd)
    assert_close(got, ref, "denoised latent")
    assert_close(got - z0, ref - z0, "latent change over the loop")


def test_denoise_one_step_equals_the_pieces():
    """One step of h3dit_denoise is the same computation as the per-piece
    entry points in sequence (embedding, h3dit_step, time embedding, output
    modulation, output layer + Euler) with fp32 tokens: equal up to the
    order-independent fp32 rounding of the shared kernels (bit-exact is
    expected; a 1e-6 relative slack is allowed)."""
    from image_generation_b200 import h3dit as H

    dims, tw, bws, io, x_txt, z0 = _denoise_case(2, 0.5)
    D = dims.hidden
    cfg = H.make_config(D, dims.heads, dims.head_dim, dims.ffn, 2, 288, io_fp32=True)
    ctx = H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws])
    dev = {k: to_dev(v, "f32") for k, v in io.items()}
    za = to_dev(z0, "f32")
    ctx.denoise(dev, za, to_dev(x_txt, "f32"), 1)
    zb = to_dev(z0, "f32")
    txt = to_dev(x_txt, "f32")
    img = torch.empty(256, D, device="cuda")
    c = torch.empty(D, device="cuda")
    mod = torch.empty(2 * D, device="cuda")
    ctx.embed_latent(zb, dev["w_in"], dev["b_in"], img)
    ctx.step(1.0, img, [(0, 16, 16)], txt)
    ctx.time_embed(1.0, c)
    ctx.output_modulation(c, dev["w_mod"], dev["b_mod"], mod)
    ctx.output_euler(img, mod, dev["w_out"], dev["b_out"], zb, -1.0)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    a, b = to_np(za), to_np(zb)
    assert np.abs(a - b).max() <= 1e-6 * np.abs(b).max()


def test_denoise_argument_errors():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    ctx, _, _ = _ctx(dims, max_tokens=64)
    D = dims.hidden
    io = {k: to_dev(v, "f32") for k, v in _io(D, 24, 14).items()}
    z = torch.zeros(24, 16, 16, device="cuda")       # 64 image tokens
    txt = torch.zeros(8, D, device="cuda", dtype=torch.bfloat16)
    for steps in (0, 1001):
        with pytest.raises(H.H3DitError) as e:
            ctx.denoise(io, z, None, steps)
        assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    with pytest.raises(H.H3DitError) as e:   # 64 + 8 tokens > max_tokens
        ctx.denoise(io, z, txt, 6)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    assert ctx.sync_status() == 0
