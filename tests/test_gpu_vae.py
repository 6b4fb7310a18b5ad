"""GPU parity of the image VAE's ViT decoder (shape level) through the C ABI
against oracle/vae_decoder.py on the same seeded weights: each stage
(LayerNorm, the biased linears, attention batched over tiles), the whole
decoder at a small width, and the full 24-layer decoder (W 1280, 32 x 32
tiles) on sampled tiles, which the oracle decodes independently."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import vae_decoder as V
from tests.helpers import (assert_attention_bound, assert_bf16_rounding, assert_close, to_dev,
                           to_np)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MATRICES = ("w_qkv", "w_o", "w_1", "w_2", "w_out")


def _dev(w: dict) -> dict:
    out = {k: to_dev(v, "bf16" if k in MATRICES else "f32") for k, v in w.items() if k != "layers"}
    if "layers" in w:
        out["layers"] = [_dev(l) for l in w["layers"]]
    return out


def _ocfg(v: synth.VaeDims) -> V.VaeConfig:
    return V.VaeConfig(width=v.width, heads=v.heads, head_dim=v.head_dim, mlp=v.mlp,
                       layers=v.layers, tile=v.tile, channels=v.channels)


def _decoder(v: synth.VaeDims, max_tokens: int, seed=0):
    from image_generation_b200 import h3dit as H

    w = synth.vae_weights(v, seed)
    cfg = H.make_vae_config(v.width, v.heads, v.head_dim, v.mlp, v.layers, v.tile, v.channels,
                            max_tokens)
    return H.VaeDecoder(cfg, _dev(w)), w


@pytest.fixture(scope="module")
def small():
    return _decoder(synth.VAE_SMALL, 2048)


def _ok(ctx):
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0


@pytest.mark.parametrize("n", [1, 7, 300])
def test_layernorm(small, n):
    ctx, w = small
    W = synth.VAE_SMALL.width
    x = synth.normal_f32((n, W), 2.0, n, "x") + 0.7
    g, b = w["layers"][0]["ln1_g"], w["layers"][0]["ln1_b"]
    out = torch.empty(n, W, dtype=torch.bfloat16, device="cuda")
    ctx.layernorm(to_dev(x, "f32"), to_dev(g, "f32"), to_dev(b, "f32"), out)
    _ok(ctx)
    assert_bf16_rounding(to_np(out), V.layer_norm(x, g, b, 1e-6), "layernorm", abs_floor=1e-4)


@pytest.mark.parametrize("m", [1, 130, 300])
def test_linear_with_bias(small, m):
    from image_generation_b200 import h3dit as H

    ctx, _ = small
    k, n = 256, 800
    a = synth.tokens(m, k, m, "a")
    wt = synth.normal_bf16((n, k), 0.05, m, "w")
    b = synth.normal_f32((n,), 0.5, m, "b")
    ref = V.affine(a, wt, b)
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ctx.linear_bias(H.H3DIT_EPI_STORE, to_dev(a), to_dev(wt), to_dev(b, "f32"), out)
    _ok(ctx)
    assert_bf16_rounding(to_np(out), ref, "linear + bias", abs_floor=1e-3)
    ctx.linear_bias(H.H3DIT_EPI_GELU, to_dev(a), to_dev(wt), to_dev(b, "f32"), out)
    _ok(ctx)
    assert_bf16_rounding(to_np(out), V.gelu(ref), "linear + bias + GELU", abs_floor=1e-3)
    x = synth.normal_f32((m, n), 1.0, m, "x")
    gate = np.ones(n, np.float32)
    xd = to_dev(x, "f32")
    ctx.linear_bias(H.H3DIT_EPI_GATED_RESIDUAL, to_dev(a), to_dev(wt), to_dev(b, "f32"), xd,
                    gate=to_dev(gate, "f32"))
    _ok(ctx)
    assert_close(to_np(xd) - x, ref, "residual + linear + bias", cos_min=0.999999, rel_max=1e-4)


@pytest.mark.parametrize("n,batch", [(256, 3), (100, 4), (1024, 2)])
def test_attention_batched(small, n, batch):
    """Each sequence of the batch attends only to its own tokens; a ragged
    length (100) has query tiles and key tiles that run past it into the next
    sequence's rows, which must not be read as keys or written as output."""
    ctx, _ = small
    H, d = synth.VAE_SMALL.heads, synth.VAE_SMALL.head_dim
    I = H * d
    qkv = synth.normal_bf16((batch * n, 3 * I), 1.0, n + batch, "qkv")
    o = torch.full((batch * n, I), float("nan"), device="cuda", dtype=torch.bfloat16)
    q = to_dev(qkv)
    ctx.attention_batched(q[:, :I], q[:, I:2 * I], q[:, 2 * I:], 3 * I, o, I, n, batch)
    _ok(ctx)
    got = to_np(o)
    for z in range(batch):
        rows = slice(z * n, (z + 1) * n)
        sq = lambda c: qkv[rows, c * I:(c + 1) * I].reshape(n, H, d)
        ref = V.attention(sq(0), sq(1), sq(2)).reshape(n, I)
        assert_attention_bound(got[rows], ref, float(np.abs(sq(2)).max()), f"sequence {z}")


def test_decode_small_matches_oracle(small):
    """The whole decoder at width 256 (2 layers, 16 x 16 tiles) on a 32 x 48
    latent: six tiles decoded at once."""
    ctx, w = small
    z = synth.normal_f32((24, 32, 48), 1.0, 5, "z")
    img = torch.empty(3, 512, 768, device="cuda")
    ctx.decode(to_dev(z, "f32"), img)
    _ok(ctx)
    ref = V.decode(z, w, _ocfg(synth.VAE_SMALL))
    assert_close(to_np(img), ref, "decoded image")


def test_decode_full_size_sampled_tiles():
    """The full decoder (W 1280, 10 heads x 128, MLP 5120, 24 layers, 32 x 32
    tiles) on a 64 x 64 latent (a 1024^2 image, four tiles); the oracle decodes
    the first and the last tile on their own."""
    v = synth.VAE
    ctx, w = _decoder(v, 4096, seed=1)
    z = synth.normal_f32((24, 64, 64), 1.0, 6, "z")
    img = torch.empty(3, 1024, 1024, device="cuda")
    ctx.decode(to_dev(z, "f32"), img)
    _ok(ctx)
    got = to_np(img)
    cfg = _ocfg(v)
    for r0, c0 in ((0, 0), (32, 32)):
        ref = V.decode_tile(z[:, r0:r0 + 32, c0:c0 + 32], w, cfg)
        assert_close(got[:, 16 * r0:16 * r0 + 512, 16 * c0:16 * c0 + 512], ref,
                     f"tile at latent ({r0}, {c0})")


def test_decode_writes_only_the_image_and_rejects_bad_shapes(small):
    from image_generation_b200 import h3dit as H
    from tests.test_gpu_guards import Guarded

    ctx, _ = small
    z = to_dev(synth.normal_f32((24, 16, 32), 1.0, 7, "z"), "f32")
    img = Guarded((3, 256, 512), torch.float32)
    ctx.decode(z, img.t)
    img.check("decoded image")
    assert not bool(torch.isnan(img.t).any())
    with pytest.raises(H.H3DitError) as e:   # 20 is not a multiple of the 16-pixel tile
        ctx.decode(torch.zeros(24, 16, 20, device="cuda"), img.t)
    assert e.value.status == H.H3DIT_ERR_UNSUPPORTED
    with pytest.raises(H.H3DitError) as e:   # a DiT call on a decoder context
        ctx.time_embed(0.5, torch.empty(256, device="cuda"))
    assert e.value.status == H.H3DIT_ERR_UNSUPPORTED
    _ok(ctx)


@pytest.mark.parametrize("n", [1, 300])
def test_layernorm_wide_rows(n):
    """Rows wider than 2048 take the one-CTA-per-row form (a full-width DiT
    context, width 5376)."""
    from image_generation_b200 import h3dit as H
    from tests.helpers import time_tensors

    d = synth.FULL_96
    bw = {k: torch.zeros(16, device="cuda", dtype=torch.bfloat16)
          for k in ("w_qkv", "w_o", "w_ff1", "w_ff2", "w_ada")}
    bw["b_ada"] = torch.zeros(16, device="cuda")
    ctx = H.Context(H.make_config(d.hidden, d.heads, d.head_dim, d.ffn, 1, 16),
                    time_tensors(synth.time_weights(d, 0)), [bw])
    x = synth.normal_f32((n, d.hidden), 2.0, n, "xw") - 0.4
    g = (1.0 + synth.normal_f32((d.hidden,), 0.1, n, "g")).astype(np.float32)
    b = synth.normal_f32((d.hidden,), 0.1, n, "b")
    out = torch.empty(n, d.hidden, dtype=torch.bfloat16, device="cuda")
    ctx.layernorm(to_dev(x, "f32"), to_dev(g, "f32"), to_dev(b, "f32"), out)
    _ok(ctx)
    assert_bf16_rounding(to_np(out), V.layer_norm(x, g, b, 1e-6), "wide layernorm", abs_floor=1e-4)
