"""Pins for the CPU oracle, checked against things other than the oracle itself:
closed forms, textbook values, brute force on tiny inputs, invariants of the
method, and independently written library compositions (torch float64).

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a swapped chunk) makes it fail.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import dit_block as O
from image_generation_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f64 = torch.float64


def _tiny_cfg(head_dim=96, **kw):
    return O.config_for(hidden=48, heads=2, head_dim=head_dim, ffn=64, **kw)


def _tiny_weights(cfg, seed=1, std=0.2):
    g = np.random.default_rng(seed)
    D, I, Fh = cfg.hidden, cfg.inner, cfg.ffn
    return {
        "w_qkv": g.normal(0, std, (3 * I, D)),
        "w_o": g.normal(0, std, (D, I)),
        "w_ff1": g.normal(0, std, (Fh, D)),
        "w_ff2": g.normal(0, std, (D, Fh)),
        "w_ada": g.normal(0, std, (6 * D, D)),
        "b_ada": g.normal(0, std, (6 * D,)),
    }


# ---------------------------------------------------------------- golden shapes

def test_golden_architecture_matches_workloads():
    with open(os.path.join(GOLDEN, "architecture.json")) as fh:
        g = json.load(fh)
    d = synth.FULL_96
    assert d.hidden == g["hidden"]["value"]
    assert d.heads == g["heads"]["value"]
    assert d.ffn == g["ffn"]["value"]
    assert synth.N_BLOCKS == g["layers"]["value"]
    assert synth.N_STEPS == g["steps"]["value"]
    assert synth.FULL_128.head_dim == g["head_dim_apxml"]["value"]
    assert d.hidden // d.heads == d.head_dim  # the other reading, 5376 / 56
    assert g["vae_downsample"]["value"] * g["patch"]["value"] == g["pixels_per_token"]["value"]
    # the packed 4096^2 canvas has the printed token count
    pos = O.token_positions(0, synth.WORKLOADS["block_4k"].grids)
    assert pos.shape[0] == g["tokens_4096_canvas"]["value"]
    assert synth.WORKLOADS["block_4k"].n_tokens == 512 + 16384
    assert synth.WORKLOADS["edit_4ref"].n_tokens == 20736


# ------------------------------------------------------------ timestep (a1, a2)

def test_timestep_embedding_at_zero_is_ones_then_zeros():
    e = O.timestep_embedding(0.0)
    assert e.shape == (256,)
    assert np.array_equal(e, np.concatenate([np.ones(128), np.zeros(128)]))


def test_timestep_embedding_known_channels():
    t = 0.3
    e = O.timestep_embedding(t)
    # channel 0 has frequency 1; channel 64 has 10000^(-1/2) = 1/100
    assert e[0] == pytest.approx(math.cos(1000 * t), abs=1e-13)
    assert e[128] == pytest.approx(math.sin(1000 * t), abs=1e-13)
    assert e[64] == pytest.approx(math.cos(10 * t), abs=1e-13)
    assert e[128 + 64] == pytest.approx(math.sin(10 * t), abs=1e-13)
    assert np.allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-14)
    # frequencies strictly decrease: cos of a tiny angle is near 1 at the end
    assert e[127] == pytest.approx(math.cos(1000 * t * 10000 ** (-127 / 128)), abs=1e-13)


def test_silu_and_gelu_values():
    x = np.linspace(-6, 6, 101)
    assert np.allclose(O.silu(x), F.silu(torch.tensor(x, dtype=f64)).numpy(), atol=1e-15)
    assert O.gelu(np.array([0.0]))[0] == 0.0
    # Phi(1) from the normal table
    assert O.gelu(np.array([1.0]))[0] == pytest.approx(0.8413447460685429, abs=1e-15)
    # GELU(x) - GELU(-x) = x  (x Phi(x) + x Phi(-x) = x)
    assert np.allclose(O.gelu(x) - O.gelu(-x), x, atol=1e-14)
    assert np.allclose(O.gelu(x), F.gelu(torch.tensor(x, dtype=f64)).numpy(), atol=1e-14)
    assert np.allclose(O.gelu(x, tanh=True),
                       F.gelu(torch.tensor(x, dtype=f64), approximate="tanh").numpy(), atol=1e-14)
    assert np.max(np.abs(O.gelu(x) - O.gelu(x, tanh=True))) < 1e-3


def test_time_mlp_and_adaln_against_linear_layers():
    g = np.random.default_rng(3)
    D = 40
    w1, b1 = g.normal(size=(D, 256)), g.normal(size=D)
    w2, b2 = g.normal(size=(D, D)), g.normal(size=D)
    wa, ba = g.normal(size=(6 * D, D)), g.normal(size=6 * D)
    e = O.timestep_embedding(0.7)
    c = O.time_mlp(e, w1, b1, w2, b2)
    T = lambda a: torch.tensor(a, dtype=f64)
    c_ref = F.linear(F.silu(F.linear(T(e), T(w1), T(b1))), T(w2), T(b2))
    assert np.allclose(c, c_ref.numpy(), rtol=1e-12, atol=1e-12)
    mod = O.adaln_modulation(c, wa, ba)
    mod_ref = F.linear(F.silu(c_ref), T(wa), T(ba)).view(6, D)
    assert mod.shape == (6, D)
    assert np.allclose(mod, mod_ref.numpy(), rtol=1e-12, atol=1e-12)
    # chunk k is rows [k D, (k+1) D) of W_ada
    assert np.allclose(mod[2], wa[2 * D:3 * D] @ O.silu(c) + ba[2 * D:3 * D])


# ------------------------------------------------------------ RMSNorm (a3, a7)

def test_rms_norm_closed_forms():
    g = np.random.default_rng(4)
    x = g.normal(size=(7, 33)) * 3.0
    y = O.rms_norm(x, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=1)), 1.0, atol=1e-14)
    assert np.allclose(O.rms_norm(5.5 * x, 0.0), y, atol=1e-14)
    ref = F.rms_norm(torch.tensor(x, dtype=f64), (33,), eps=1e-6).numpy()
    assert np.allclose(O.rms_norm(x, 1e-6), ref, atol=1e-14)


def test_modulate_scale_minus_one_gives_shift():
    g = np.random.default_rng(5)
    x = g.normal(size=(9, 16))
    s = g.normal(size=16)
    xm = O.norm_modulate(x, s, -np.ones(16), 1e-6)
    assert np.array_equal(xm, np.broadcast_to(s, xm.shape))
    # identity modulation is the plain norm
    assert np.array_equal(O.norm_modulate(x, 0 * s, 0 * s, 1e-6), O.rms_norm(x, 1e-6))


# ------------------------------------------------------------------------ RoPE

def _rope_complex(x, pos, sections, theta):
    """RoPE as complex multiplication: pair j of axis a is the complex number
    x[o+j] + i x[o+s+j], multiplied by exp(i pos_a theta^(-j/s))."""
    x = torch.tensor(x, dtype=f64)
    out = x.clone()
    o = 0
    for a, s in enumerate(sections):
        j = torch.arange(s, dtype=f64)
        ang = torch.tensor(pos[:, a], dtype=f64)[:, None] * (theta ** (-j / s))[None, :]
        z = torch.complex(x[..., o:o + s], x[..., o + s:o + 2 * s])
        z = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
        out[..., o:o + s] = z.real
        out[..., o + s:o + 2 * s] = z.imag
        o += 2 * s
    return out.numpy()


@pytest.mark.parametrize("head_dim", [96, 128])
def test_rope_against_complex_rotation(head_dim):
    g = np.random.default_rng(6)
    sec = O.default_sections(head_dim)
    pos = g.integers(0, 130, size=(11, 3))
    x = g.normal(size=(11, 3, head_dim))
    assert np.allclose(O.apply_rope(x, pos, sec, 10000.0), _rope_complex(x, pos, sec, 10000.0),
                       atol=1e-12)


@pytest.mark.parametrize("head_dim", [96, 128])
def test_rope_identity_norm_and_relative_position(head_dim):
    g = np.random.default_rng(7)
    sec = O.default_sections(head_dim)
    x = g.normal(size=(5, 2, head_dim))
    zero = np.zeros((5, 3), np.int64)
    assert np.array_equal(O.apply_rope(x, zero, sec, 1e4), x)
    pos = g.integers(0, 64, size=(5, 3))
    y = O.apply_rope(x, pos, sec, 1e4)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)
    # <R(m) q, R(n) k> depends only on m - n, per axis
    q, k = g.normal(size=(1, 1, head_dim)), g.normal(size=(1, 1, head_dim))
    m, n = np.array([[1, 5, 9]]), np.array([[0, 2, 30]])
    base = np.sum(O.apply_rope(q, m, sec, 1e4) * O.apply_rope(k, n, sec, 1e4))
    for shift in ([3, 0, 0], [0, 7, 0], [0, 0, 11], [2, 40, 17]):
        sft = np.array([shift])
        got = np.sum(O.apply_rope(q, m + sft, sec, 1e4) * O.apply_rope(k, n + sft, sec, 1e4))
        assert got == pytest.approx(base, abs=1e-11)
    # moving along one axis only touches that axis' channels
    p1 = np.array([[0, 0, 5]])
    y = O.apply_rope(q, p1, sec, 1e4)
    lo = 2 * (sec[0] + sec[1])
    assert np.array_equal(y[..., :lo], q[..., :lo])
    assert not np.allclose(y[..., lo:], q[..., lo:])


def test_token_positions_layout():
    pos = O.token_positions(3, [(0, 2, 3), (2, 1, 2)])
    assert pos.shape == (3 + 6 + 2, 3)
    assert np.array_equal(pos[:3], np.zeros((3, 3)))
    assert pos[3:9].tolist() == [[0, 0, 0], [0, 0, 1], [0, 0, 2], [0, 1, 0], [0, 1, 1], [0, 1, 2]]
    assert pos[9:].tolist() == [[2, 0, 0], [2, 0, 1]]


# ------------------------------------------------------------------- attention

def _attention_loops(q, k, v):
    R, H, d = q.shape
    N = k.shape[0]
    out = np.zeros((R, H, d))
    for r, h in itertools.product(range(R), range(H)):
        s = [sum(q[r, h, c] * k[n, h, c] for c in range(d)) / math.sqrt(d) for n in range(N)]
        mx = max(s)
        p = [math.exp(si - mx) for si in s]
        z = sum(p)
        for c in range(d):
            out[r, h, c] = sum(p[n] * v[n, h, c] for n in range(N)) / z
    return out


def test_attention_brute_force_and_library():
    g = np.random.default_rng(8)
    q, k, v = (g.normal(size=(6, 2, 4)) * 2 for _ in range(3))
    o = O.attention(q, k, v)
    assert np.allclose(o, _attention_loops(q, k, v), atol=1e-13)
    T = lambda a: torch.tensor(a, dtype=f64).transpose(0, 1)[None]
    ref = F.scaled_dot_product_attention(T(q), T(k), T(v))[0].transpose(0, 1).numpy()
    assert np.allclose(o, ref, atol=1e-13)


def test_attention_degenerate_cases():
    g = np.random.default_rng(9)
    q = g.normal(size=(3, 2, 8))
    v1 = g.normal(size=(1, 2, 8))
    assert np.allclose(O.attention(q, g.normal(size=(1, 2, 8)), v1), np.broadcast_to(v1, (3, 2, 8)))
    k_same = np.broadcast_to(g.normal(size=(1, 2, 8)), (5, 2, 8))
    v = g.normal(size=(5, 2, 8))
    assert np.allclose(O.attention(q, k_same, v), np.broadcast_to(v.mean(0), (3, 2, 8)), atol=1e-14)


# ----------------------------------------------------------------- whole block

def _textbook_block(x, w, pos, cfg, sh1, sc1, g1, sh2, sc2, g2):
    """A pre-norm block with AdaLN written from torch library calls, with the
    modulation vectors passed by name."""
    T = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    X = T(x)
    N, D = X.shape
    H, d, I = cfg.heads, cfg.head_dim, cfg.inner
    h = F.rms_norm(X, (D,), eps=cfg.norm_eps) * (1 + T(sc1)) + T(sh1)
    q, k, v = F.linear(h, T(w["w_qkv"])).split(I, dim=-1)
    q = T(_rope_complex(q.reshape(N, H, d).numpy(), pos, cfg.rope_sections, cfg.rope_theta))
    k = T(_rope_complex(k.reshape(N, H, d).numpy(), pos, cfg.rope_sections, cfg.rope_theta))
    v = v.reshape(N, H, d)
    a = F.scaled_dot_product_attention(q.transpose(0, 1)[None], k.transpose(0, 1)[None],
                                       v.transpose(0, 1)[None])[0].transpose(0, 1).reshape(N, I)
    X = X + T(g1) * F.linear(a, T(w["w_o"]))
    h = F.rms_norm(X, (D,), eps=cfg.norm_eps) * (1 + T(sc2)) + T(sh2)
    act = F.gelu(F.linear(h, T(w["w_ff1"])), approximate="tanh" if cfg.gelu_tanh else "none")
    return (X + T(g2) * F.linear(act, T(w["w_ff2"]))).numpy()


def _tiny_case(head_dim=96, n_txt=4, grids=((0, 3, 4),), seed=11, **kw):
    cfg = _tiny_cfg(head_dim, **kw)
    w = _tiny_weights(cfg, seed)
    pos = O.token_positions(n_txt, grids)
    g = np.random.default_rng(seed + 100)
    x = g.normal(size=(pos.shape[0], cfg.hidden))
    return cfg, w, pos, x, g


@pytest.mark.parametrize("head_dim,gelu_tanh", [(96, False), (128, False), (96, True)])
def test_block_against_textbook_with_named_modulation(head_dim, gelu_tanh):
    cfg, w, pos, x, g = _tiny_case(head_dim, gelu_tanh=gelu_tanh)
    D = cfg.hidden
    sh1, sc1, g1, sh2, sc2, g2 = (g.normal(size=D) * 0.5 for _ in range(6))
    mod = np.stack([sh1, sc1, g1, sh2, sc2, g2])
    y = O.block_forward(x, mod, w, pos, cfg)
    ref = _textbook_block(x, w, pos, cfg, sh1, sc1, g1, sh2, sc2, g2)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-11)


def test_identity_adaln_is_plain_prenorm_block():
    cfg, w, pos, x, g = _tiny_case()
    D = cfg.hidden
    z, one = np.zeros(D), np.ones(D)
    y = O.block_forward(x, np.stack([z, z, one, z, z, one]), w, pos, cfg)
    ref = _textbook_block(x, w, pos, cfg, z, z, one, z, z, one)
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-11)


def test_zero_gates_return_input_exactly():
    cfg, w, pos, x, g = _tiny_case()
    mod = g.normal(size=(6, cfg.hidden))
    mod[2] = 0.0
    mod[5] = 0.0
    assert np.array_equal(O.block_forward(x, mod, w, pos, cfg), x)


def test_sampled_rows_equal_full_rows():
    cfg, w, pos, x, g = _tiny_case(grids=((0, 4, 5),))
    mod = g.normal(size=(6, cfg.hidden)) * 0.3
    full = O.block_forward(x, mod, w, pos, cfg)
    rows = [0, 3, 7, 23]
    assert np.allclose(O.block_forward(x, mod, w, pos, cfg, rows=rows), full[rows], atol=1e-13)


def test_text_permutation_equivariance():
    cfg, w, pos, x, g = _tiny_case(n_txt=5)
    mod = g.normal(size=(6, cfg.hidden)) * 0.3
    y = O.block_forward(x, mod, w, pos, cfg)
    perm = np.array([3, 0, 4, 1, 2])
    xp = x.copy()
    xp[:5] = x[perm]
    yp = O.block_forward(xp, mod, w, pos, cfg)
    assert np.allclose(yp[:5], y[perm], atol=1e-12)
    assert np.allclose(yp[5:], y[5:], atol=1e-12)


def test_grid_shift_invariance_without_text():
    cfg, w, pos, x, g = _tiny_case(n_txt=0, grids=((0, 3, 3), (1, 2, 3)))
    x = x[: pos.shape[0]]
    mod = g.normal(size=(6, cfg.hidden)) * 0.3
    y = O.block_forward(x, mod, w, pos, cfg)
    y2 = O.block_forward(x, mod, w, pos + np.array([2, 5, 9]), cfg)
    assert np.allclose(y, y2, atol=1e-11)


def test_image_permutation_with_positions():
    cfg, w, pos, x, g = _tiny_case(n_txt=2, grids=((0, 3, 3),))
    mod = g.normal(size=(6, cfg.hidden)) * 0.3
    y = O.block_forward(x, mod, w, pos, cfg)
    perm = np.concatenate([[0, 1], 2 + g.permutation(9)])
    yp = O.block_forward(x[perm], mod, w, pos[perm], cfg)
    assert np.allclose(yp, y[perm], atol=1e-12)


def test_step_is_adaln_once_then_blocks_in_order():
    cfg, w0, pos, x, g = _tiny_case()
    w1 = _tiny_weights(cfg, seed=99)
    tw = {"w_t1": g.normal(size=(cfg.hidden, 256)) * 0.1, "b_t1": g.normal(size=cfg.hidden),
          "w_t2": g.normal(size=(cfg.hidden, cfg.hidden)) * 0.1, "b_t2": g.normal(size=cfg.hidden)}
    t = 0.4
    y = O.step_forward(x, t, tw, [w0, w1], pos, cfg)
    T = lambda a: torch.tensor(a, dtype=f64)
    e = T(O.timestep_embedding(t))
    c = F.linear(F.silu(F.linear(e, T(tw["w_t1"]), T(tw["b_t1"]))), T(tw["w_t2"]), T(tw["b_t2"]))
    ref = x
    for w in (w0, w1):
        m = F.linear(F.silu(c), T(w["w_ada"]), T(w["b_ada"])).view(6, -1).numpy()
        ref = _textbook_block(ref, w, pos, cfg, *m)
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-10)


def test_flop_count_matches_linear_shapes():
    # count multiply-adds of each product the block performs, at a small size
    n, D, H, d, Fh = 37, 48, 2, 96, 64
    I = H * d
    macs = n * D * 3 * I + n * I * D + n * D * Fh + n * Fh * D + H * (n * n * d) * 2
    assert O.block_flops(n, D, I, Fh) == 2 * macs


# ---------------------------------------------------------------- MXFP8 (a11)

def _all_e4m3_values():
    """Every finite E4M3 value, enumerated from the bit fields."""
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # the NaN code
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.add(v)
            vals.add(-v)
    return np.array(sorted(vals))


def test_e4m3_rounding_is_nearest_representable():
    grid = _all_e4m3_values()
    assert grid.max() == 448.0 and len(grid) == 253  # 127 positive, 127 negative, one zero
    assert np.array_equal(O.e4m3_round(grid), grid)  # representable values are fixed
    g = np.random.default_rng(12)
    x = np.concatenate([g.normal(size=4000) * 50, g.uniform(-500, 500, 2000), [1e-9, -3e-3]])
    q = O.e4m3_round(x)
    assert np.all(np.isin(q, grid))
    inside = np.abs(x) <= 448
    # nearest: no representable value is strictly closer
    dist = np.abs(grid[None, :] - x[inside, None]).min(axis=1)
    assert np.allclose(np.abs(q[inside] - x[inside]), dist, atol=0)
    assert np.all(q[~inside] == np.sign(x[~inside]) * 448.0)  # saturation
    # ties go to the even mantissa: 1 + 1/16 lies between 1 and 1.125
    assert O.e4m3_round(np.array([1.0625, 1.1875, -1.0625]))[0] == 1.0
    assert O.e4m3_round(np.array([1.1875]))[0] == 1.25
    normal = (np.abs(x) >= 2.0 ** -6) & inside
    assert np.max(np.abs(q[normal] - x[normal]) / np.abs(x[normal])) <= 2.0 ** -4


def test_mx_quantize_scales_and_roundtrip():
    g = np.random.default_rng(13)
    x = g.normal(size=(5, 96)) * np.array([1e-3, 1.0, 300.0])[np.arange(96) // 32]
    q, X = O.mx_quantize(x)
    assert X.shape == (5, 3) and np.array_equal(X, np.floor(X))
    blocks = np.abs(x).reshape(5, 3, 32).max(axis=2)
    # the block maximum lands in [256, 512) before rounding, so its code is in [256, 448]
    assert np.all((blocks / 2.0 ** X >= 256) & (blocks / 2.0 ** X < 512))
    qmax = np.abs(q).reshape(5, 3, 32).max(axis=2)
    assert np.all((qmax >= 256) & (qmax <= 448))
    y = O.mx_dequantize(q, X)
    big = np.abs(x) >= 2.0 ** (np.repeat(X, 32, axis=1) - 6)
    assert np.max(np.abs(y - x)[big] / np.abs(x)[big]) <= 2.0 ** -4
    # values already on the grid survive exactly
    exact = np.repeat(2.0 ** X, 32, axis=1) * O.e4m3_round(g.uniform(-400, 400, (5, 96)))
    assert np.array_equal(O.mx_roundtrip(exact), exact)
    zq, zX = O.mx_quantize(np.zeros((1, 32)))
    assert np.all(zq == 0) and zX[0, 0] == -127


def test_mx_linear_and_block_reduce_to_bf16_block_on_grid_values():
    """If every operand is already exactly representable in MXFP8, the MXFP8
    linear equals the plain one."""
    g = np.random.default_rng(14)
    x = O.e4m3_round(g.uniform(-300, 300, (7, 64))) * 2.0 ** -5
    w = O.e4m3_round(g.uniform(-300, 300, (9, 64))) * 2.0 ** -9
    assert np.allclose(O.linear_mx(x, w), O.linear(x, w), rtol=0, atol=1e-12)
    cfg = O.config_for(hidden=64, heads=2, head_dim=96, ffn=64)
    wb = _tiny_weights(cfg, seed=15)
    pos = O.token_positions(3, [(0, 3, 4)])
    g2 = np.random.default_rng(16)
    xb = g2.normal(size=(pos.shape[0], cfg.hidden))
    mod = g2.normal(size=(6, cfg.hidden)) * 0.3
    y_mx = O.block_forward_mx(xb, mod, wb, pos, cfg)
    y = O.block_forward(xb, mod, wb, pos, cfg)
    d_mx, d = y_mx - xb, y - xb
    cos = np.sum(d_mx * d) / np.linalg.norm(d_mx) / np.linalg.norm(d)
    assert 0.99 < cos < 1.0  # close to, but not the same as, the unquantized block
    mod[2] = mod[5] = 0.0
    assert np.array_equal(O.block_forward_mx(xb, mod, wb, pos, cfg), xb)
