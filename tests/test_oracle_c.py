"""The two oracles against each other: the numpy float64 oracle
(oracle/dit_block.py) and the independent plain-C one (oracle/h3ref.c), in
its double build to rounding level and in its float build (the block in plain
fp32) to the accuracy fp32 accumulation allows. Both were written from the
pages; a mistake in either (a dropped term, a wrong sign, a transposed
operand) shows up as a mismatch here. CPU only."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from oracle import ref_c


@pytest.fixture(scope="module")
def refs(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("h3ref"))
    ref_c.build(d)
    return {k: ref_c.RefC(ref_c.lib_path(k, d)) for k in ("f64", "f32")}


def _rel(a, b):
    return float(np.abs(np.asarray(a, np.float64) - b).max() / np.abs(b).max())


def _cos(a, b):
    a, b = np.asarray(a, np.float64).ravel(), np.asarray(b, np.float64).ravel()
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def test_builds_use_their_arithmetic_type(refs):
    assert refs["f64"].real is np.float64 and refs["f32"].real is np.float32


@pytest.mark.parametrize("n_txt,grids", [(0, [(0, 4, 5)]), (3, [(0, 5, 7), (1, 3, 4), (3, 2, 9)])])
def test_token_positions_agree(refs, n_txt, grids):
    assert np.array_equal(refs["f64"].token_positions(n_txt, grids), O.token_positions(n_txt, grids))


@pytest.mark.parametrize("t", [0.0, 0.37, 1.0])
def test_timestep_condition_and_adaln_agree(refs, t):
    d = synth.Dims(hidden=192, heads=2, head_dim=96, ffn=256)
    tw = synth.time_weights(d, 3)
    tw["b_t1"] = synth.normal_f32((d.hidden,), 0.1, 3, "b_t1")
    tw["b_t2"] = synth.normal_f32((d.hidden,), 0.1, 3, "b_t2")
    cfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
    c_ref = O.timestep_condition(t, tw, cfg)
    for kind, tol in (("f64", 1e-12), ("f32", 2e-5)):
        c = refs[kind].timestep_condition(t, tw)
        assert _rel(c, c_ref) < tol, kind
    w_ada = synth.normal_bf16((6 * d.hidden, d.hidden), 0.05, 4, "w_ada")
    b_ada = synth.normal_f32((6 * d.hidden,), 0.1, 4, "b_ada")
    mod_ref = O.adaln_modulation(c_ref, w_ada, b_ada)
    assert _rel(refs["f64"].adaln(c_ref, w_ada, b_ada), mod_ref) < 1e-12


def _case(dims, n_txt, grids, seed, mod_std=0.3):
    n = n_txt + sum(h * w for _, h, w in grids)
    x = synth.tokens(n, dims.hidden, seed, "x")
    w = synth.block_weights(dims, seed)
    mod = synth.normal_f32((6, dims.hidden), mod_std, seed, "mod")
    return x, w, mod, O.token_positions(n_txt, grids)


@pytest.mark.parametrize("dims,n_txt,grids,tanh", [
    (synth.SMALL, 32, [(0, 16, 16)], False),                       # the small workload, d_h 96
    (synth.Dims(256, 2, 128, 512), 5, [(0, 6, 7), (2, 3, 5)], False),  # d_h 128, two frames
    (synth.Dims(192, 2, 96, 384), 4, [(0, 5, 6)], True),           # the tanh GELU
], ids=["small_d96", "d128_frames", "gelu_tanh"])
def test_block_forward_agrees(refs, dims, n_txt, grids, tanh):
    x, w, mod, pos = _case(dims, n_txt, grids, 11)
    cfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn, gelu_tanh=tanh)
    ref = O.block_forward(x, mod, w, pos, cfg)
    kw = dict(heads=dims.heads, head_dim=dims.head_dim, sections=cfg.rope_sections, gelu_tanh=tanh)
    y64 = refs["f64"].block_forward(x, mod, w, pos, **kw)
    assert _rel(y64, ref) < 1e-11
    assert _rel(y64 - x, ref - x) < 1e-10  # the branch delta, not hidden by the residual
    y32 = refs["f32"].block_forward(x, mod, w, pos, **kw)
    delta = ref - x
    assert _cos(y32 - x, delta) > 0.999999
    assert np.abs(y32 - ref).max() < 1e-4 * np.sqrt(np.mean(delta ** 2)) + 1e-5 * np.abs(ref).max()


def test_zero_gates_return_the_input_exactly(refs):
    """Both gates zero: y = x bit for bit, in the float build too."""
    dims = synth.Dims(192, 2, 96, 384)
    x, w, mod, pos = _case(dims, 3, [(0, 4, 4)], 5)
    mod[2] = 0.0
    mod[5] = 0.0
    cfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    for kind in ("f64", "f32"):
        y = refs[kind].block_forward(x, mod, w, pos, heads=2, head_dim=96, sections=cfg.rope_sections)
        assert np.array_equal(y, x.astype(refs[kind].real)), kind


def test_sections_must_cover_head_dim(refs):
    dims = synth.Dims(192, 2, 96, 384)
    x, w, mod, pos = _case(dims, 2, [(0, 2, 2)], 6)
    with pytest.raises(AssertionError):
        refs["f64"].block_forward(x, mod, w, pos, heads=2, head_dim=96, sections=(16, 16, 8))


# Mistakes of the kinds a hand-written block gets wrong, planted in a copy of
# the C source: each must move the output past the cross-check's tolerance.
PLANTED = {
    "rope sign": ("v[o + j] = x1 * cs - x2 * sn;", "v[o + j] = x1 * cs + x2 * sn;"),
    "rope pair": ("x2 = v[o + s + j];", "x2 = v[o + s - 1 - j];"),
    "modulate without 1 +": ("* ((REAL)1 + scale[j]) + shift[j]", "* scale[j] + shift[j]"),
    "attention scale off by 1%": ("p[j] = s * scale;", "p[j] = s * scale * (REAL)1.01;"),
    "gates swapped": ("y[i] = x1[i] + g2[i % D] * t[i];", "y[i] = x1[i] + g1[i % D] * t[i];"),
    "rmsnorm eps dropped": ("R_SQRT(ss / (REAL)d + (REAL)eps)", "R_SQRT(ss / (REAL)d)"),
    "K from the Q rows": ("linear(xm, n, D, w_qkv + (size_t)I * D, I, k);",
                          "linear(xm, n, D, w_qkv, I, k);"),
    "softmax not normalised": ("const REAL w = p[j] / sum;", "const REAL w = p[j];"),
    "GELU erf argument unscaled": ("R_ERF(x / (REAL)1.4142135623730951)", "R_ERF(x)"),
}


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_cross_check_catches_planted_mistake(tmp_path, name):
    old, new = PLANTED[name]
    src = open(ref_c.SRC).read()
    assert old in src
    path = tmp_path / "h3ref.c"
    path.write_text(src.replace(old, new))
    ref_c.build(str(tmp_path), src=str(path), werror=False)
    bad = ref_c.RefC(ref_c.lib_path("f64", str(tmp_path)))
    dims = synth.Dims(192, 2, 96, 384)
    x, w, mod, pos = _case(dims, 4, [(0, 5, 6)], 13)
    cfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    ref = O.block_forward(x, mod, w, pos, cfg)
    y = bad.block_forward(x, mod, w, pos, heads=2, head_dim=96, sections=cfg.rope_sections)
    assert _rel(y, ref) > 1e-9, f"{name} went unnoticed"
