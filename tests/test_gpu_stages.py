"""Parity of each step of the path, through the C ABI, against the oracle on the
same seeded inputs: sizes span several tiles and ragged tails (rows that are
not a multiple of 128, a single row)."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import (assert_attention_bound, assert_bf16_rounding, assert_close,
                           block_tensors, time_tensors, to_dev, to_np)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _make(dims: synth.Dims, n_blocks=2, max_tokens=1100, seed=0):
    from image_generation_b200 import h3dit as H

    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, max_tokens)
    tw = synth.time_weights(dims, seed)
    bws = [synth.block_weights(dims, seed + 1000 + l) for l in range(n_blocks)]
    ctx = H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws])
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    return ctx, ocfg, tw, bws


@pytest.fixture(scope="module")
def small():
    return _make(synth.SMALL)


@pytest.fixture(scope="module")
def small128():
    # head_dim 128 at a small width: 6 heads x 128 = 768 attention channels
    return _make(synth.Dims(hidden=768, heads=6, head_dim=128, ffn=2048))


def _ok(ctx):
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0


@pytest.mark.parametrize("t", [0.0, 0.5, 0.913])
def test_time_embed_and_adaln(small, t):
    ctx, ocfg, tw, bws = small
    D = ocfg.hidden
    c = torch.empty(D, dtype=torch.float32, device="cuda")
    ctx.time_embed(t, c)
    mod = torch.empty(2, 6, D, dtype=torch.float32, device="cuda")
    c_ref = O.timestep_condition(t, tw, ocfg)
    # feed the oracle's c to the projection so the two steps are checked apart
    ctx.adaln_project(to_dev(c_ref, "f32"), 0, 2, mod)
    _ok(ctx)
    assert_close(to_np(c), c_ref, "time embed", cos_min=0.999999, rel_max=1e-4)
    for l in range(2):
        ref = O.adaln_modulation(c_ref, bws[l]["w_ada"], bws[l]["b_ada"])
        assert_close(to_np(mod[l]), ref, f"adaln block {l}", cos_min=0.999999, rel_max=1e-4)


@pytest.mark.parametrize("n", [1, 7, 300])
def test_rmsnorm_modulate(small, n):
    ctx, ocfg, _, _ = small
    D = ocfg.hidden
    x = synth.normal_f32((n, D), 1.5, 7, "x") + 0.3
    sh = synth.normal_f32((D,), 0.3, 7, "shift")
    sc = synth.normal_f32((D,), 0.3, 7, "scale")
    out = torch.empty(n, D, dtype=torch.bfloat16, device="cuda")
    ctx.rmsnorm_modulate(to_dev(x, "f32"), to_dev(sh, "f32"), to_dev(sc, "f32"), out)
    _ok(ctx)
    ref = O.norm_modulate(x, sh, sc, ocfg.norm_eps)
    assert_bf16_rounding(to_np(out), ref, "rmsnorm+modulate")


def test_rmsnorm_modulate_extreme_rows(small):
    """Rows of exact zeros (the epsilon alone sets the scale: the output is
    the shift), rows near the bottom of fp32 (squares below the smallest
    normal) and rows near its top (squares summed near 1e33): the kernel's
    fp32 sum of squares must neither overflow nor flush a row to zero where
    the float64 oracle does not."""
    ctx, ocfg, _, _ = small
    D = ocfg.hidden
    x = synth.normal_f32((8, D), 1.0, 8, "x")
    x[0] = 0.0
    x[1] *= np.float32(1e-20)
    x[2] *= np.float32(1e15)
    x[3, :] = 0.0
    x[3, 5] = np.float32(3e-30)  # a single tiny nonzero
    sh = synth.normal_f32((D,), 0.3, 8, "shift")
    sc = synth.normal_f32((D,), 0.3, 8, "scale")
    out = torch.empty(8, D, dtype=torch.bfloat16, device="cuda")
    ctx.rmsnorm_modulate(to_dev(x, "f32"), to_dev(sh, "f32"), to_dev(sc, "f32"), out)
    _ok(ctx)
    got = to_np(out)
    ref = O.norm_modulate(x.astype(np.float64), sh, sc, ocfg.norm_eps)
    assert np.all(np.isfinite(got))
    assert_bf16_rounding(got, ref, "rmsnorm+modulate, extreme rows")
    assert np.array_equal(got[0], to_np(to_dev(sh)))  # zero row: exactly the shift in bf16


@pytest.mark.parametrize("grids,n_txt", [([(0, 16, 16)], 32), ([(0, 5, 7), (1, 3, 4), (3, 2, 9)], 3),
                                         ([(0, 128, 128)], 512)])
@pytest.mark.parametrize("which", ["small", "small128"])
def test_rope_table(request, grids, n_txt, which):
    ctx, ocfg, _, _ = request.getfixturevalue(which)
    pos = O.token_positions(n_txt, grids)
    n = pos.shape[0]
    table = torch.empty(n, ocfg.head_dim // 2, 2, dtype=torch.float32, device="cuda")
    ctx.rope_table(grids, n_txt, table)
    _ok(ctx)
    ang = O.rope_angles(pos, ocfg.rope_sections, ocfg.rope_theta)
    got = to_np(table)
    assert np.max(np.abs(got[..., 0] - np.cos(ang))) < 2e-6
    assert np.max(np.abs(got[..., 1] - np.sin(ang))) < 2e-6


def _linear_case(m, n, k, seed):
    a = synth.tokens(m, k, seed, "a")
    w = synth.normal_bf16((n, k), 0.02, seed, "w")
    return a, w


@pytest.mark.parametrize("m", [1, 130, 300, 520])
@pytest.mark.parametrize("n,k", [(768, 768), (2048, 768), (768, 2048), (800, 768)])
def test_linear_store_and_gelu(small, m, n, k):
    from image_generation_b200 import h3dit as H

    ctx, ocfg, _, _ = small
    a, w = _linear_case(m, n, k, m + n + k)
    ref = O.linear(a, w)
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ctx.linear(H.H3DIT_EPI_STORE, to_dev(a), to_dev(w), out)
    _ok(ctx)
    assert_bf16_rounding(to_np(out), ref, "linear", abs_floor=1e-3)
    assert_close(to_np(out), ref, "linear")
    out.zero_()
    ctx.linear(H.H3DIT_EPI_GELU, to_dev(a), to_dev(w), out)
    _ok(ctx)
    assert_close(to_np(out), O.gelu(ref), "linear+gelu")
    # the epilogue's erf (Abramowitz & Stegun 7.1.26, |error| <= 1.5e-7) keeps
    # GELU within one bf16 rounding of the exact erf form
    assert_bf16_rounding(to_np(out), O.gelu(ref), "linear+gelu", abs_floor=1e-3)


@pytest.mark.parametrize("k", [64, 192])
def test_linear_several_tiles_per_cta(small, k):
    """More output tiles than CTAs: each persistent CTA (or CTA pair) runs
    several tiles through both TMEM accumulators; a ragged last row block and
    a short K (one k-block is fewer than the ring's stages)."""
    from image_generation_b200 import h3dit as H

    ctx, _, _, _ = small
    m, n = 4500, 4096
    a, w = _linear_case(m, n, k, 5 + k)
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ctx.linear(H.H3DIT_EPI_STORE, to_dev(a), to_dev(w), out)
    _ok(ctx)
    assert_bf16_rounding(to_np(out), O.linear(a, w), "linear", abs_floor=1e-3)


@pytest.mark.parametrize("m", [1, 257])
def test_linear_gated_residual(small, m):
    from image_generation_b200 import h3dit as H

    ctx, ocfg, _, _ = small
    n, k = 768, 2048
    a, w = _linear_case(m, n, k, 11)
    x = synth.normal_f32((m, n), 1.0, 11, "x")
    gate = synth.normal_f32((n,), 0.3, 11, "gate")
    xt = to_dev(x, "f32")
    ctx.linear(H.H3DIT_EPI_GATED_RESIDUAL, to_dev(a), to_dev(w), xt, gate=to_dev(gate, "f32"))
    _ok(ctx)
    ref = x + gate * O.linear(a, w)
    assert_close(to_np(xt), ref, "gated residual", cos_min=0.9999999, rel_max=1e-4)
    assert_close((to_np(xt) - x).ravel(), (ref - x).ravel(), "gated residual delta")


@pytest.mark.parametrize("which", ["small", "small128"])
@pytest.mark.parametrize("n_txt,grids", [(32, [(0, 16, 16)]), (3, [(0, 5, 7), (2, 9, 11)])])
def test_linear_qkv_rope(request, which, n_txt, grids):
    from image_generation_b200 import h3dit as H

    ctx, ocfg, _, bws = request.getfixturevalue(which)
    pos = O.token_positions(n_txt, grids)
    m = pos.shape[0]
    xm = synth.tokens(m, ocfg.hidden, 5, "xm")
    table = torch.empty(m, ocfg.head_dim // 2, 2, dtype=torch.float32, device="cuda")
    ctx.rope_table(grids, n_txt, table)
    out = torch.empty(m, 3 * ocfg.inner, dtype=torch.bfloat16, device="cuda")
    ctx.linear(H.H3DIT_EPI_QKV_ROPE, to_dev(xm), to_dev(bws[0]["w_qkv"]), out, rope_table=table)
    _ok(ctx)
    q, k, v = O.qkv_rope(xm, bws[0]["w_qkv"], pos, ocfg)
    ref = np.concatenate([q.reshape(m, -1), k.reshape(m, -1), v.reshape(m, -1)], axis=1)
    got = to_np(out)
    assert_close(got, ref, "qkv+rope")
    assert_bf16_rounding(got, ref, "qkv+rope", abs_floor=1e-3)


@pytest.mark.parametrize("which", ["small", "small128"])
@pytest.mark.parametrize("n", [1, 100, 128, 300, 1000])
@pytest.mark.parametrize("packed", [True, False])
def test_attention(request, which, n, packed):
    ctx, ocfg, _, _ = request.getfixturevalue(which)
    H_, d = ocfg.heads, ocfg.head_dim
    I = H_ * d
    q = synth.normal_bf16((n, H_, d), 1.5, n, "q")
    k = synth.normal_bf16((n, H_, d), 1.5, n, "k")
    v = synth.normal_bf16((n, H_, d), 1.0, n, "v")
    if packed:
        qkv = to_dev(np.concatenate([q.reshape(n, I), k.reshape(n, I), v.reshape(n, I)], axis=1))
        qt, kt, vt, ld = qkv[:, :I], qkv[:, I:2 * I], qkv[:, 2 * I:], 3 * I
    else:
        qt, kt, vt, ld = to_dev(q.reshape(n, I)), to_dev(k.reshape(n, I)), to_dev(v.reshape(n, I)), I
    o = torch.empty(n, I, dtype=torch.bfloat16, device="cuda")
    ctx.attention(qt, kt, vt, ld, o, I, n)
    _ok(ctx)
    ref = O.attention(q, k, v).reshape(n, I)
    assert_attention_bound(to_np(o), ref, float(np.abs(v).max()), "attention")


def _rescales_per_row(q, k, d, bkv=64, threshold=8.0):
    """How often the kernel's running max is replaced (and O rescaled) per
    query row: the max starts at the first 64-key tile's row max, in log2
    units, and moves only when a tile's max exceeds it by more than 8."""
    n, H_ = q.shape[0], q.shape[1]
    sl2 = np.log2(np.e) / np.sqrt(d)
    counts = np.zeros((n, H_), np.int64)
    for h in range(H_):
        s = (q[:, h].astype(np.float64) @ k[:, h].astype(np.float64).T) * sl2
        m = s[:, :bkv].max(axis=1)
        for j in range(bkv, s.shape[1], bkv):
            mx = s[:, j:j + bkv].max(axis=1)
            grow = mx > m + threshold
            counts[grow, h] += 1
            m = np.where(grow, mx, m)
    return counts


@pytest.mark.parametrize("which", ["small", "small128"])
@pytest.mark.parametrize("pattern", ["jump", "gradual"])
def test_attention_running_max_growth(request, which, pattern):
    """Scores that grow along the key sequence, so that the running max moves
    by more than 8 (log2 units) and O is rescaled in tensor memory: a shared
    component in dimension 0 of every head (q + 4, k + 24 from key 500 on:
    one jump of 12-14 log2 units; or k + 3 t in key tile t: a rescale every
    few tiles). Without the rescale the early keys would weigh up to 2^8
    times too much, far outside the bound."""
    ctx, ocfg, _, _ = request.getfixturevalue(which)
    H_, d = ocfg.heads, ocfg.head_dim
    I, n = H_ * d, 1000
    q = synth.normal_bf16((n, H_, d), 1.0, 11, "q").astype(np.float32)
    k = synth.normal_bf16((n, H_, d), 1.0, 11, "k").astype(np.float32)
    v = synth.normal_bf16((n, H_, d), 1.0, 11, "v")
    q[:, :, 0] += 4.0
    if pattern == "jump":
        k[500:, :, 0] += 24.0
    else:
        k[:, :, 0] += 3.0 * (np.arange(n) // 64)[:, None]
    q, k = synth.round_to_bf16(q), synth.round_to_bf16(k)  # the values the GPU sees
    counts = _rescales_per_row(q, k, d)
    # the case does what it is for: (almost) every row's O gets rescaled
    assert (counts >= 1).mean() > 0.9, float((counts >= 1).mean())
    if pattern == "gradual":
        assert counts.mean() > 1.5, float(counts.mean())
    o = torch.empty(n, I, dtype=torch.bfloat16, device="cuda")
    ctx.attention(to_dev(q.reshape(n, I)), to_dev(k.reshape(n, I)), to_dev(v.reshape(n, I)), I, o,
                  I, n)
    _ok(ctx)
    ref = O.attention(q, k, v).reshape(n, I)
    assert_attention_bound(to_np(o), ref, float(np.abs(v).max()), f"attention, {pattern} max")


def test_attention_identical_keys_give_mean_of_values(small):
    ctx, ocfg, _, _ = small
    n, H_, d = 300, ocfg.heads, ocfg.head_dim
    I = H_ * d
    q = synth.normal_bf16((n, H_, d), 1.0, 3, "q")
    k = np.broadcast_to(synth.normal_bf16((1, H_, d), 1.0, 3, "k"), (n, H_, d))
    v = synth.normal_bf16((n, H_, d), 1.0, 3, "v")
    o = torch.empty(n, I, dtype=torch.bfloat16, device="cuda")
    ctx.attention(to_dev(q.reshape(n, I)), to_dev(k.reshape(n, I)), to_dev(v.reshape(n, I)), I, o, I, n)
    _ok(ctx)
    mean = np.broadcast_to(v.astype(np.float64).mean(0).reshape(1, I), (n, I))
    assert_close(to_np(o), mean, "attention of identical keys")
