"""Out-of-bounds write checks for every entry point (in place of a memory
sanitizer): each output, and each context's workspace, sits inside a larger
buffer whose margins before and after are filled with 0xFF bytes - NaN as
bf16, fp32 and E4M3 - and after ragged calls (rows that are not a multiple of
the tiles, a single row, token counts past a tile boundary) every margin byte
must still be 0xFF. Attention writes into rows with a stride wider than its
output, so a store past the last head of a row is caught too. The values
themselves are checked by the parity tests; this file only looks at bytes the
library must not touch."""
import numpy as np
import pytest

from image_generation_b200 import synth
from tests.helpers import block_tensors, time_tensors, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MARGIN = 64 * 1024  # bytes of 0xFF on each side (a multiple of 256: keeps the view aligned)


class Guarded:
    """A tensor of `shape` and `dtype` placed between two 0xFF margins."""

    def __init__(self, shape, dtype, init=None):
        self.nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        body = (self.nbytes + 255) // 256 * 256
        self.buf = torch.full((2 * MARGIN + body,), 0xFF, dtype=torch.uint8, device="cuda")
        self.t = self.buf[MARGIN:MARGIN + self.nbytes].view(dtype).view(*shape)
        if init is not None:
            self.t.copy_(init)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.buf[:MARGIN]
        tail = self.buf[MARGIN + self.nbytes:]
        bad_head = int((head != 0xFF).sum())
        bad_tail = int((tail != 0xFF).sum())
        assert bad_head == 0 and bad_tail == 0, (
            f"{what}: {bad_head} bytes changed before the buffer, {bad_tail} after it")


def _context(dims, n_blocks=1, max_tokens=1100, precision=0, io_fp32=False, seed=0):
    """A context on seeded weights whose workspace is itself guarded."""
    from image_generation_b200 import h3dit as H

    import ctypes as C

    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, max_tokens,
                        precision=precision, io_fp32=io_fp32)
    ws = Guarded((int(H.lib.h3dit_workspace_bytes(C.byref(cfg))),), torch.uint8)
    tw = synth.time_weights(dims, seed)
    bws = [synth.block_weights(dims, seed + 1000 + l) for l in range(n_blocks)]
    ctx = H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws], workspace=ws.t)
    return ctx, ws, bws


@pytest.fixture(scope="module")
def bf16_ctx():
    return _context(synth.SMALL, n_blocks=2)


@pytest.fixture(scope="module")
def mx_ctx():
    from image_generation_b200 import h3dit as H

    return _context(synth.SMALL, n_blocks=1, precision=H.H3DIT_PRECISION_MXFP8)


def _ok(ctx, ws, what):
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    ws.check(what + " (workspace)")


def _rope_for(ctx, m, head_dim):
    """A RoPE table for m tokens: one text token per row past a 2-row grid."""
    table = torch.empty(m, head_dim // 2, 2, device="cuda")
    grids = [(0, 2, m // 2)] if m >= 2 else []
    ctx.rope_table(grids, m - 2 * (m // 2) if m >= 2 else m, table)
    return table


@pytest.mark.parametrize("m", [1, 130, 257])
def test_linear_epilogues(bf16_ctx, m):
    from image_generation_b200 import h3dit as H

    ctx, ws, _ = bf16_ctx
    D, I = synth.SMALL.hidden, synth.SMALL.inner
    a = to_dev(synth.tokens(m, D, m, "a"))
    w800 = to_dev(synth.normal_bf16((800, D), 0.02, m, "w"))
    for epi in (H.H3DIT_EPI_STORE, H.H3DIT_EPI_GELU):
        out = Guarded((m, 800), torch.bfloat16)
        ctx.linear(epi, a, w800, out.t)
        out.check(f"linear epilogue {epi}, m={m}, n=800")
    wqkv = to_dev(synth.normal_bf16((3 * I, D), 0.02, m, "wqkv"))
    table = _rope_for(ctx, m, synth.SMALL.head_dim)
    out = Guarded((m, 3 * I), torch.bfloat16)
    ctx.linear(H.H3DIT_EPI_QKV_ROPE, a, wqkv, out.t, rope_table=table)
    out.check(f"QKV + RoPE, m={m}")
    x = Guarded((m, D), torch.float32, init=torch.randn(m, D, device="cuda"))
    gate = torch.full((D,), 0.25, device="cuda")
    wo = to_dev(synth.normal_bf16((D, 832), 0.02, m, "wo"))   # k = 13 k-blocks of 64
    a832 = to_dev(synth.tokens(m, 832, m, "a832"))
    ctx.linear(H.H3DIT_EPI_GATED_RESIDUAL, a832, wo, x.t, gate=gate)
    x.check(f"gated residual, m={m}")
    _ok(ctx, ws, f"linear m={m}")


@pytest.mark.parametrize("dh", [96, 128])
@pytest.mark.parametrize("n", [1, 100, 1000])
def test_attention(n, dh):
    dims = synth.SMALL if dh == 96 else synth.Dims(hidden=768, heads=6, head_dim=128, ffn=2048)
    ctx, ws, _ = _context(dims)
    I = dims.inner
    qkv = torch.randn(n, 3 * I, device="cuda").bfloat16()
    gap = 64  # columns between one row's last head and the next row
    o = Guarded((n, I + gap), torch.bfloat16)
    ctx.attention(qkv[:, :I], qkv[:, I:2 * I], qkv[:, 2 * I:], 3 * I, o.t, I + gap, n)
    o.check(f"attention n={n} d_h={dh}")
    torch.cuda.synchronize()
    untouched = o.t[:, I:].contiguous().view(torch.uint8)
    assert bool((untouched == 0xFF).all()), "attention wrote into the columns past heads*head_dim"
    assert not bool(torch.isnan(o.t[:, :I].float()).any()), "attention left output elements unwritten"
    _ok(ctx, ws, f"attention n={n}")


@pytest.mark.parametrize("n", [1, 7, 300])
def test_rmsnorm_time_adaln_rope(bf16_ctx, n):
    ctx, ws, _ = bf16_ctx
    D = synth.SMALL.hidden
    x = torch.randn(n, D, device="cuda")
    sh = torch.randn(D, device="cuda") * 0.1
    sc = torch.randn(D, device="cuda") * 0.1
    out = Guarded((n, D), torch.bfloat16)
    ctx.rmsnorm_modulate(x, sh, sc, out.t)
    out.check(f"rmsnorm n={n}")
    c = Guarded((D,), torch.float32)
    ctx.time_embed(0.3, c.t)
    c.check("time embed")
    mod = Guarded((1, 6, D), torch.float32)
    ctx.adaln_project(c.t, 1, 1, mod.t)
    mod.check("adaln projection of one block")
    grids = [(0, 5, 7), (1, 3, 4)]
    table = Guarded((n + 47, 48, 2), torch.float32)
    ctx.rope_table(grids, n, table.t)
    table.check("rope table")
    _ok(ctx, ws, f"rmsnorm/time/adaln/rope n={n}")


@pytest.mark.parametrize("io_fp32", [False, True], ids=["bf16_tokens", "fp32_tokens"])
def test_block_forward_and_step(io_fp32):
    dims = synth.SMALL
    D = dims.hidden
    ctx, ws, _ = _context(dims, n_blocks=2, max_tokens=300, io_fp32=io_fp32)
    dt = torch.float32 if io_fp32 else torch.bfloat16
    grids = [(0, 5, 7), (1, 3, 4), (2, 16, 13)]
    n_img = 35 + 12 + 208
    txt = Guarded((3, D), dt, init=torch.randn(3, D, device="cuda").to(dt))
    img = Guarded((n_img, D), dt, init=torch.randn(n_img, D, device="cuda").to(dt))
    ctx.block_forward(1, 0.4, img.t, grids, txt.t)
    txt.check("block_forward text tokens")
    img.check("block_forward image tokens")
    ctx.step(0.7, img.t, grids, txt.t)
    txt.check("step text tokens")
    img.check("step image tokens")
    _ok(ctx, ws, "block and step")


@pytest.mark.parametrize("m", [1, 130, 257])
def test_mxfp8_entry_points(mx_ctx, m):
    from image_generation_b200 import h3dit as H

    ctx, ws, _ = mx_ctx
    dims = synth.SMALL
    D, I, F = dims.hidden, dims.inner, dims.ffn
    # quantize: dst and scales
    src = torch.randn(m, D, device="cuda").bfloat16()
    aq = Guarded((m, D), torch.uint8)
    asf = Guarded((H.mx_scale_bytes(m, D),), torch.uint8)
    ctx.mx_quantize(src, aq.t, asf.t)
    aq.check(f"mx quantize m={m}")
    asf.check(f"mx quantize scales m={m}")
    # the block's four MXFP8 linears through the step's kernels
    table = _rope_for(ctx, m, dims.head_dim)
    out = Guarded((m, 3 * I), torch.bfloat16)
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_QKV, aq.t, asf.t, out.t, rope_table=table)
    out.check(f"MXFP8 QKV m={m}")
    x = Guarded((m, D), torch.float32, init=torch.randn(m, D, device="cuda"))
    gate = torch.full((D,), 0.25, device="cuda")
    oq = torch.zeros(m, I, dtype=torch.uint8, device="cuda")
    osf = torch.full((H.mx_scale_bytes(m, I),), 127, dtype=torch.uint8, device="cuda")
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_OUT, oq, osf, x.t, gate=gate)
    x.check(f"MXFP8 out-projection m={m}")
    u = Guarded((m, F), torch.uint8)
    usf = Guarded((H.mx_scale_bytes(m, F),), torch.uint8)
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_FFN1, aq.t, asf.t, u.t, out_sf=usf.t)
    u.check(f"MXFP8 FFN1 m={m}")
    usf.check(f"MXFP8 FFN1 scales m={m}")
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_FFN2, u.t, usf.t, x.t, gate=gate)
    x.check(f"MXFP8 FFN2 m={m}")
    # the public MXFP8 linear with the standard scale layout, STORE epilogue
    wq = torch.empty(512, D, dtype=torch.uint8, device="cuda")
    wsf = torch.empty(H.mx_scale_bytes(512, D), dtype=torch.uint8, device="cuda")
    ctx.mx_quantize(torch.randn(512, D, device="cuda").bfloat16() * 0.02, wq, wsf)
    o2 = Guarded((m, 512), torch.bfloat16)
    ctx.linear_mx(H.H3DIT_EPI_STORE, aq.t, asf.t, wq, wsf, o2.t)
    o2.check(f"MXFP8 linear m={m}")
    # the MXFP8 norm and attention outputs
    xr = torch.randn(m, D, device="cuda")
    z = torch.zeros(D, device="cuda")
    nq = Guarded((m, D), torch.uint8)
    nsf = Guarded((H.mx_scale_bytes(m, D),), torch.uint8)
    ctx.rmsnorm_modulate_mx(xr, z, z, nq.t, nsf.t)
    nq.check(f"MXFP8 rmsnorm m={m}")
    nsf.check(f"MXFP8 rmsnorm scales m={m}")
    qkv = torch.randn(m, 3 * I, device="cuda").bfloat16()
    aoq = Guarded((m, I), torch.uint8)
    aosf = Guarded((H.mx_scale_bytes(m, I),), torch.uint8)
    ctx.attention_mx(qkv[:, :I], qkv[:, I:2 * I], qkv[:, 2 * I:], 3 * I, aoq.t, aosf.t, m)
    aoq.check(f"MXFP8 attention m={m}")
    aosf.check(f"MXFP8 attention scales m={m}")
    _ok(ctx, ws, f"MXFP8 m={m}")


def test_mxfp8_step():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    D = dims.hidden
    ctx, ws, _ = _context(dims, n_blocks=2, max_tokens=300, precision=H.H3DIT_PRECISION_MXFP8)
    grids = [(0, 16, 16), (1, 1, 3)]
    txt = Guarded((5, D), torch.bfloat16, init=torch.randn(5, D, device="cuda").bfloat16())
    img = Guarded((259, D), torch.bfloat16, init=torch.randn(259, D, device="cuda").bfloat16())
    ctx.step(0.5, img.t, grids, txt.t)
    txt.check("MXFP8 step text tokens")
    img.check("MXFP8 step image tokens")
    _ok(ctx, ws, "MXFP8 step")


@pytest.mark.parametrize("shape", [(24, 18, 26), (3, 4, 6)], ids=["24x18x26", "3x4x6"])
def test_io_layers_and_denoise(shape):
    dims = synth.SMALL
    D = dims.hidden
    ctx, ws, _ = _context(dims, n_blocks=1, max_tokens=300, io_fp32=False)
    C, Hl, Wl = shape
    n = (Hl // 2) * (Wl // 2)
    f = lambda s, tag: torch.from_numpy(synth.normal_f32(s, 0.05, 3, tag)).cuda()
    io = {"w_in": f((D, 4 * C), "w_in"), "b_in": f((D,), "b_in"), "w_mod": f((2 * D, D), "w_mod"),
          "b_mod": f((2 * D,), "b_mod"), "w_out": f((4 * C, D), "w_out"),
          "b_out": f((4 * C,), "b_out")}
    z = Guarded(shape, torch.float32, init=torch.randn(*shape, device="cuda"))
    x = Guarded((n, D), torch.bfloat16)
    ctx.embed_latent(z.t, io["w_in"], io["b_in"], x.t)
    x.check("patch embedding")
    c = torch.randn(D, device="cuda")
    mod = Guarded((2 * D,), torch.float32)
    ctx.output_modulation(c, io["w_mod"], io["b_mod"], mod.t)
    mod.check("output modulation")
    ctx.output_euler(x.t, mod.t, io["w_out"], io["b_out"], z.t, -0.25)
    z.check("output layer + Euler")
    txt = Guarded((7, D), torch.bfloat16, init=torch.randn(7, D, device="cuda").bfloat16())
    ctx.denoise(io, z.t, txt.t, 2)
    z.check("denoise latent")
    txt.check("denoise text tokens")
    _ok(ctx, ws, "io layers")


def test_time_embed_static():
    from image_generation_b200 import h3dit as H

    D = 768
    tw = {k: to_dev(v, "f32") for k, v in synth.time_weights(synth.SMALL, 4).items()}
    c = Guarded((D,), torch.float32)
    st = H.lib.h3dit_time_embed_static(tw["w_t1"].data_ptr(), tw["b_t1"].data_ptr(),
                                       tw["w_t2"].data_ptr(), tw["b_t2"].data_ptr(), D, 0.5,
                                       1000.0, c.t.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == H.H3DIT_OK
    c.check("static time embed")


@pytest.mark.parametrize("P", [2, 4])
def test_sequence_parallel_relayouts(bf16_ctx, P):
    ctx, ws, _ = bf16_ctx
    I = synth.SMALL.inner
    n = 37  # rows of one rank, not a multiple of anything
    qkv = torch.randn(n, 3 * I, device="cuda").bfloat16()
    send = Guarded((P, n, 3 * I // P), torch.bfloat16)
    ctx.sp_pack_qkv(qkv, P, send.t)
    send.check(f"sequence-parallel pack, {P} ranks")
    recv = torch.randn(P, n, I // P, device="cuda").bfloat16()
    o = Guarded((n, I), torch.bfloat16)
    ctx.sp_unpack_o(recv, P, o.t)
    o.check(f"sequence-parallel unpack, {P} ranks")
    heads = synth.SMALL.heads // P
    q = torch.randn(P * n, 3 * I // P, device="cuda").bfloat16()
    cw = I // P
    oh = Guarded((P * n, cw + 16), torch.bfloat16)   # rows wider than the head group
    ctx.attention_heads(heads, q[:, :cw], q[:, cw:2 * cw], q[:, 2 * cw:], 3 * cw, oh.t, cw + 16,
                        P * n)
    oh.check(f"attention on {heads} heads")
    torch.cuda.synchronize()
    assert bool((oh.t[:, cw:].contiguous().view(torch.uint8) == 0xFF).all())
    _ok(ctx, ws, f"sequence-parallel {P}")


@pytest.mark.parametrize("m", [1, 130, 257])
def test_decoder_stage_entry_points(m):
    from image_generation_b200 import h3dit as H

    import ctypes as C

    v = synth.VAE_SMALL
    cfg = H.make_vae_config(v.width, v.heads, v.head_dim, v.mlp, v.layers, v.tile, v.channels,
                            2048)
    ws = Guarded((int(H.lib.h3dit_vae_workspace_bytes(C.byref(cfg))),), torch.uint8)
    w = synth.vae_weights(v, 0)
    dev = {k: to_dev(val, "bf16" if k == "w_out" else "f32") for k, val in w.items()
           if k != "layers"}
    mats = ("w_qkv", "w_o", "w_1", "w_2")
    dev["layers"] = [{k: to_dev(val, "bf16" if k in mats else "f32") for k, val in l.items()}
                     for l in w["layers"]]
    ctx = H.VaeDecoder(cfg, dev, workspace=ws.t)
    W = v.width
    x = torch.randn(m, W, device="cuda")
    ln = Guarded((m, W), torch.bfloat16)
    ctx.layernorm(x, dev["lnf_g"], dev["lnf_b"], ln.t)
    ln.check(f"layernorm m={m}")
    wt = torch.randn(800, W, device="cuda").bfloat16()
    b = torch.randn(800, device="cuda")
    for epi in (H.H3DIT_EPI_STORE, H.H3DIT_EPI_GELU):
        out = Guarded((m, 800), torch.bfloat16)
        ctx.linear_bias(epi, ln.t, wt, b, out.t)
        out.check(f"linear + bias, epilogue {epi}, m={m}")
    res = Guarded((m, 800), torch.float32, init=torch.randn(m, 800, device="cuda"))
    ctx.linear_bias(H.H3DIT_EPI_GATED_RESIDUAL, ln.t, wt, b, res.t,
                    gate=torch.ones(800, device="cuda"))
    res.check(f"residual + linear + bias, m={m}")
    I = v.heads * v.head_dim
    q = torch.randn(3 * m, 3 * I, device="cuda").bfloat16()
    o = Guarded((3 * m, I), torch.bfloat16)
    ctx.attention_batched(q[:, :I], q[:, I:2 * I], q[:, 2 * I:], 3 * I, o.t, I, m, 3)
    o.check(f"attention over 3 sequences of {m}")
    _ok(ctx, ws, f"decoder stages m={m}")
