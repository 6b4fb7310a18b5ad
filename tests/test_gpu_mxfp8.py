"""Parity of the MXFP8 variant (a11) through the C ABI against the oracle's
OCP-MX reading. Weight quantization is integer work on exactly representable
inputs, so it is compared bit for bit. Outputs written as MXFP8 are held to
the E4M3 rounding bound per element; whole blocks to the MXFP8 tolerance,
cosine >= 0.999 (on the output and on the branch delta): the GPU quantizes
fp32 activations and the oracle float64 ones, so an element can land on the
other side of a rounding boundary, which a max-abs bound would not allow."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import (assert_attention_bound, assert_close, assert_delta_close,
                           block_tensors, time_tensors, to_dev, to_np)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

MX_COS = 0.999


def assert_mx_bound(codes, X, ref, what, extra=None):
    """An MXFP8 output is the reference rounded to E4M3 (nearest even,
    saturating at 448) under its block scale 2^X. Without `extra`, the GPU
    quantized an fp32 value within rounding noise of `ref`, so the codes must
    equal the reference's rounding except for rare one-ulp flips at rounding
    midpoints. With `extra` (error already in the value that was quantized),
    each element must be within one E4M3 ulp plus `extra` of that rounding.
    Either way the cosine must be >= 0.999."""
    got = O.mx_dequantize(codes, X)
    ref = np.asarray(ref, np.float64)
    cos = float(np.sum(got * ref) / (np.linalg.norm(got) * np.linalg.norm(ref)))
    assert cos >= MX_COS, f"{what}: cosine {cos:.6f}"
    scale = 2.0 ** np.repeat(X, 32, axis=1)
    want = O.e4m3_round(ref / scale) * scale
    one_ulp = 2.0 ** -3 * np.abs(want) + scale * 2.0 ** -9
    if extra is None:
        flips = got != want
        assert np.mean(flips) <= 1e-3, f"{what}: {np.mean(flips):.2e} of the codes differ"
        bound = one_ulp
    else:
        bound = one_ulp + 1.07 * extra
    bad = np.argwhere(np.abs(got - want) > bound * (1 + 1e-6))
    assert bad.size == 0, (f"{what}: {len(bad)} elements beyond the E4M3 bound; first {bad[0].tolist()}"
                           f" got {got[tuple(bad[0])]!r} want {want[tuple(bad[0])]!r}")


def _e4m3_table():
    """Value of every E4M3 byte, from its bit fields (0x7F / 0xFF are NaN)."""
    t = np.zeros(256)
    for b in range(256):
        sgn = -1.0 if b & 0x80 else 1.0
        e, m = (b >> 3) & 0xF, b & 7
        if e == 15 and m == 7:
            t[b] = np.nan
        elif e == 0:
            t[b] = sgn * (m / 8.0) * 2.0 ** -6
        else:
            t[b] = sgn * (1 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3 = _e4m3_table()


def _decode(q_dev, sf_dev, rows, k):
    """E4M3 codes and scale exponents X of a device MXFP8 matrix."""
    from image_generation_b200 import h3dit as H

    codes = E4M3[q_dev.cpu().numpy().astype(np.int64)].reshape(rows, k)
    sf = sf_dev.cpu().numpy()
    r = np.arange(rows)[:, None]
    s = np.arange(k // 32)[None, :]
    off = ((r // 128) * (k // 128) + s // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + s % 4
    X = sf[off].astype(np.float64) - 127.0
    return codes, X


def _alloc_mx(rows, k):
    from image_generation_b200 import h3dit as H

    q = torch.empty(rows * k, dtype=torch.uint8, device="cuda")
    sf = torch.full((H.mx_scale_bytes(rows, k),), 0, dtype=torch.uint8, device="cuda")
    return q, sf


def _ctx(dims, n_blocks=1, max_tokens=1100, precision=0, io_fp32=False, seed=0, **kw):
    from image_generation_b200 import h3dit as H

    tw = synth.time_weights(dims, seed)
    bws = [synth.block_weights(dims, seed + 1000 + l) for l in range(n_blocks)]
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, max_tokens,
                        precision=precision, io_fp32=io_fp32, **kw)
    return H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws]), tw, bws


@pytest.fixture(scope="module")
def small():
    return _ctx(synth.SMALL)[0]


@pytest.mark.parametrize("rows,k", [(300, 768), (128, 2048), (1, 128)])
def test_quantize_is_bit_exact(small, rows, k):
    g = np.random.default_rng(rows + k)
    w = synth.normal_bf16((rows, k), 0.02, rows + k, "w")
    w[0, :32] = 0.0                                   # an all-zero block
    w[rows // 2, 40] = synth.round_to_bf16(np.array([300.0], np.float32))[0]  # an outlier
    q, sf = _alloc_mx(rows, k)
    small.mx_quantize(to_dev(w), q, sf)
    torch.cuda.synchronize()
    assert small.sync_status() == 0
    codes, X = _decode(q, sf, rows, k)
    ref_q, ref_X = O.mx_quantize(w)
    assert np.array_equal(X, ref_X)
    assert np.array_equal(codes, ref_q)


def test_rmsnorm_modulate_mx(small):
    D, n = 768, 257
    x = synth.normal_f32((n, D), 1.3, 2, "x")
    sh = synth.normal_f32((D,), 0.3, 2, "sh")
    sc = synth.normal_f32((D,), 0.3, 2, "sc")
    q, sf = _alloc_mx(n, D)
    small.rmsnorm_modulate_mx(to_dev(x, "f32"), to_dev(sh, "f32"), to_dev(sc, "f32"), q, sf)
    torch.cuda.synchronize()
    assert small.sync_status() == 0
    codes, X = _decode(q, sf, n, D)
    ref = O.norm_modulate(x, sh, sc, 1e-6)
    rq, rX = O.mx_quantize(ref)
    assert np.mean(X != rX) < 1e-3          # fp32 vs fp64 can flip a scale at a power of two
    got = O.mx_dequantize(codes, X)
    assert_close(got, O.mx_dequantize(rq, rX), "rmsnorm mx vs oracle mx", cos_min=0.99999,
                 rel_max=0.2)
    assert_mx_bound(codes, X, ref, "rmsnorm mx vs unquantized oracle")


def _quantized(ctx, a):
    rows, k = a.shape
    q, sf = _alloc_mx(rows, k)
    ctx.mx_quantize(to_dev(a), q, sf)
    return q.view(rows, k), sf


@pytest.mark.parametrize("m", [1, 200, 300])
@pytest.mark.parametrize("n,k", [(768, 768), (2048, 768), (768, 2048)])
def test_linear_mx_epilogues(small, m, n, k):
    from image_generation_b200 import h3dit as H

    a = synth.tokens(m, k, m + n, "a")
    w = synth.normal_bf16((n, k), 0.02, m + n, "w")
    aq, asf = _quantized(small, a)
    wq, wsf = _quantized(small, w)
    ref = O.linear_mx(a, w)
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    small.linear_mx(H.H3DIT_EPI_STORE, aq, asf, wq, wsf, out)
    x = synth.normal_f32((m, n), 1.0, 3, "x")
    gate = synth.normal_f32((n,), 0.3, 3, "gate")
    xt = to_dev(x, "f32")
    small.linear_mx(H.H3DIT_EPI_GATED_RESIDUAL, aq, asf, wq, wsf, xt, gate=to_dev(gate, "f32"))
    uq, usf = _alloc_mx(m, n)
    small.linear_mx(H.H3DIT_EPI_GELU, aq, asf, wq, wsf, uq, out_sf=usf)
    torch.cuda.synchronize()
    assert small.sync_status() == 0
    assert_close(to_np(out), ref, "linear mx", cos_min=0.99999)
    assert_close(to_np(xt) - x, gate * ref, "linear mx gated residual", cos_min=0.99999, rel_max=1e-3)
    codes, X = _decode(uq, usf, m, n)
    assert_mx_bound(codes, X, O.gelu(ref), "linear mx gelu (MXFP8 out)")


@pytest.mark.parametrize("k", [128, 256])
def test_linear_mx_several_tiles_per_cta(small, k):
    """More output tiles than CTAs (pairs): several tiles per persistent CTA
    through both accumulators and the scale columns of every stage; a ragged
    last row block; fewer k-blocks than stages."""
    from image_generation_b200 import h3dit as H

    m, n = 4500, 2048
    a = synth.tokens(m, k, 7 + k, "a")
    w = synth.normal_bf16((n, k), 0.02, 7 + k, "w")
    aq, asf = _quantized(small, a)
    wq, wsf = _quantized(small, w)
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    small.linear_mx(H.H3DIT_EPI_STORE, aq, asf, wq, wsf, out)
    torch.cuda.synchronize()
    assert small.sync_status() == 0
    assert_close(to_np(out), O.linear_mx(a, w), "linear mx, many tiles", cos_min=0.99999)


@pytest.mark.parametrize("grids", [[(0, 9, 11)], [(0, 16, 17)]], ids=["104tok", "277tok"])
@pytest.mark.parametrize("dims", [synth.SMALL, synth.Dims(768, 6, 128, 2048)], ids=["d96", "d128"])
def test_linear_mx_qkv_rope(dims, grids):
    from image_generation_b200 import h3dit as H

    ctx, _, bws = _ctx(dims)
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    n_txt = 5
    pos = O.token_positions(n_txt, grids)
    m = pos.shape[0]
    xm = synth.tokens(m, dims.hidden, 4, "xm")
    table = torch.empty(m, dims.head_dim // 2, 2, dtype=torch.float32, device="cuda")
    ctx.rope_table(grids, n_txt, table)
    aq, asf = _quantized(ctx, xm)
    wq, wsf = _quantized(ctx, bws[0]["w_qkv"])
    out = torch.empty(m, 3 * ocfg.inner, dtype=torch.bfloat16, device="cuda")
    ctx.linear_mx(H.H3DIT_EPI_QKV_ROPE, aq, asf, wq, wsf, out, rope_table=table)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    I = ocfg.inner
    y = O.linear_mx(xm, bws[0]["w_qkv"])
    q = O.apply_rope(y[:, :I].reshape(m, -1, dims.head_dim), pos, ocfg.rope_sections, 1e4)
    k = O.apply_rope(y[:, I:2 * I].reshape(m, -1, dims.head_dim), pos, ocfg.rope_sections, 1e4)
    ref = np.concatenate([q.reshape(m, -1), k.reshape(m, -1), y[:, 2 * I:]], axis=1)
    assert_close(to_np(out), ref, "qkv mx + rope", cos_min=0.99999)


@pytest.mark.parametrize("n", [100, 1000])
def test_attention_mx_output(small, n):
    H_, d = 8, 96
    I = H_ * d
    q = synth.normal_bf16((n, H_, d), 1.5, n, "q")
    k = synth.normal_bf16((n, H_, d), 1.5, n, "k")
    v = synth.normal_bf16((n, H_, d), 1.0, n, "v")
    oq, osf = _alloc_mx(n, I)
    small.attention_mx(to_dev(q.reshape(n, I)), to_dev(k.reshape(n, I)), to_dev(v.reshape(n, I)), I,
                       oq, osf, n)
    torch.cuda.synchronize()
    assert small.sync_status() == 0
    codes, X = _decode(oq, osf, n, I)
    ref = O.attention(q, k, v).reshape(n, I)
    # the quantized O already carries the bf16 rounding of P (see assert_attention_bound)
    assert_mx_bound(codes, X, ref, "attention (MXFP8 out)",
                    extra=2.0 ** -7 * (np.abs(ref) + np.abs(v).max()))


def _block_mx_case(dims, n_txt, grids, seed, rows=None):
    w = synth.ragged(dims, n_txt, grids, seed, t=0.4)
    ctx, tw, bws = _ctx(dims, max_tokens=w.n_tokens, precision=1, io_fp32=True, seed=seed)
    inp = synth.workload_inputs(w)
    xt, xi = to_dev(inp["x_txt"], "f32"), to_dev(inp["x_img"], "f32")
    ctx.block_forward(0, w.t, xi, list(w.grids), xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    y = np.concatenate([to_np(xt), to_np(xi)], axis=0)
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    x = O.pack(inp["x_txt"], inp["x_img"])
    bw = bws[0]
    mod = O.adaln_modulation(O.timestep_condition(w.t, tw, ocfg), bw["w_ada"], bw["b_ada"])
    ref = O.block_forward_mx(x, mod, bw, O.token_positions(n_txt, w.grids), ocfg, rows=rows)
    return y if rows is None else y[rows], x if rows is None else x[rows], ref


@pytest.mark.parametrize("dims", [synth.SMALL, synth.Dims(768, 6, 128, 2048)], ids=["d96", "d128"])
def test_block_mx_small(dims):
    y, x, ref = _block_mx_case(dims, 32, [(0, 16, 16)], 8)
    assert_close(y, ref, "MXFP8 block", cos_min=MX_COS, rel_max=np.inf)
    assert_delta_close(y - x, ref - x, "MXFP8 block (branch delta)", cos_min=MX_COS, row_cos_min=0.99)


def test_block_mx_wide_tiles():
    """Hidden 2688 (28 heads x 96), FFN 3584: every linear's N is a multiple
    of 224, so the block runs all four on the wide (128 x 224) tiles with the
    W scales repacked per tile; 21 text + 18 x 17 image tokens span several
    row blocks with a ragged last one."""
    dims = synth.Dims(2688, 28, 96, 3584)
    y, x, ref = _block_mx_case(dims, 21, [(0, 18, 17)], 5)
    assert_close(y, ref, "MXFP8 block, wide tiles", cos_min=MX_COS, rel_max=np.inf)
    assert_delta_close(y - x, ref - x, "MXFP8 block, wide tiles (branch delta)", cos_min=MX_COS,
                       row_cos_min=0.99)


@pytest.mark.parametrize("dims", [synth.Dims(2688, 28, 96, 3584), synth.SMALL, synth.Dims(768, 6, 128, 2048)],
                         ids=["wide_d96", "narrow_d96", "narrow_d128"])
def test_block_linear_mx_stages(dims):
    """Each of a block's MXFP8 linears through the stage entry point, on the
    context's own quantized weights: wide (128 x 224) tiles where every N is
    a multiple of 224 (hidden 2688), the 128-wide kernel otherwise."""
    _block_linear_mx_stages(dims, [(0, 11, 19)], 9)


def test_block_linear_mx_wide_several_tiles_per_cta():
    """Hidden 2688, 1065 tokens: 9 row tiles of 128 (the last ragged) x 36
    QKV (16 FFN1, 12 out / FFN2) column tiles of 224, so with 148 CTAs each
    takes two or three tiles and both TMEM accumulators turn over."""
    _block_linear_mx_stages(synth.Dims(2688, 28, 96, 3584), [(0, 32, 33)], 9)


def _block_linear_mx_stages(dims, grids, n_txt):
    from image_generation_b200 import h3dit as H

    pos = O.token_positions(n_txt, grids)
    ctx, _, bws = _ctx(dims, max_tokens=max(300, pos.shape[0]), precision=1)
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    I, D, F = ocfg.inner, dims.hidden, dims.ffn
    bw = bws[0]
    m = pos.shape[0]
    # QKV + RoPE
    x = synth.tokens(m, D, 21, "x")
    xq, xsf = _quantized(ctx, x)
    table = torch.empty(m, dims.head_dim // 2, 2, dtype=torch.float32, device="cuda")
    ctx.rope_table(grids, n_txt, table)
    qkv = torch.empty(m, 3 * I, dtype=torch.bfloat16, device="cuda")
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_QKV, xq, xsf, qkv, rope_table=table)
    y = O.linear_mx(x, bw["w_qkv"])
    q = O.apply_rope(y[:, :I].reshape(m, -1, dims.head_dim), pos, ocfg.rope_sections, 1e4)
    k = O.apply_rope(y[:, I:2 * I].reshape(m, -1, dims.head_dim), pos, ocfg.rope_sections, 1e4)
    ref = np.concatenate([q.reshape(m, -1), k.reshape(m, -1), y[:, 2 * I:]], axis=1)
    # out-projection and FFN2 with the gated residual, FFN1 to MXFP8
    a = synth.tokens(m, I, 22, "a")
    aq, asf = _quantized(ctx, a)
    u = synth.tokens(m, F, 23, "u")
    uq, usf = _quantized(ctx, u)
    r0 = synth.normal_f32((m, D), 1.0, 24, "r")
    gate = synth.normal_f32((D,), 0.3, 24, "g")
    r_out, r_ff2 = to_dev(r0, "f32"), to_dev(r0, "f32")
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_OUT, aq, asf, r_out, gate=to_dev(gate, "f32"))
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_FFN2, uq, usf, r_ff2, gate=to_dev(gate, "f32"))
    hq, hsf = _alloc_mx(m, F)
    ctx.block_linear_mx(0, H.H3DIT_LINEAR_FFN1, xq, xsf, hq, out_sf=hsf)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    assert_close(to_np(qkv), ref, "block QKV mx + rope", cos_min=0.99999)
    assert_close(to_np(r_out) - r0, gate * O.linear_mx(a, bw["w_o"]), "block out-proj mx",
                 cos_min=0.99999, rel_max=1e-3)
    assert_close(to_np(r_ff2) - r0, gate * O.linear_mx(u, bw["w_ff2"]), "block FFN2 mx",
                 cos_min=0.99999, rel_max=1e-3)
    codes, X = _decode(hq, hsf, m, F)
    assert_mx_bound(codes, X, O.gelu(O.linear_mx(x, bw["w_ff1"])), "block FFN1 mx gelu")


def test_block_mx_full_width_4k_sampled_rows():
    w = synth.WORKLOADS["block_4k"]
    rows = np.unique(np.concatenate([np.arange(24), np.random.default_rng(3).choice(
        np.arange(512, w.n_tokens), 96, replace=False), [w.n_tokens - 1]]))
    y, x, ref = _block_mx_case(w.dims, w.n_txt, list(w.grids), 0, rows=rows)
    assert_close(y, ref, "MXFP8 block 4096^2", cos_min=MX_COS, rel_max=np.inf)
    assert_delta_close(y - x, ref - x, "MXFP8 block 4096^2 (branch delta)", cos_min=MX_COS,
                       row_cos_min=0.99)
