"""Parity at the full model width and sequence lengths of the pages' workloads
(2048^2 and 4096^2 canvases, the 4-reference edit), in the launch
configuration the benchmark times, on sampled output rows the oracle can
compute one by one (keys and values over all tokens)."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import assert_close, assert_delta_close, block_tensors, time_tensors, to_dev, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _sample_rows(n_txt, n, seed, k_img=160):
    g = np.random.default_rng(seed)
    txt = np.arange(min(n_txt, 48))
    img = g.choice(np.arange(n_txt, n), size=min(k_img, n - n_txt), replace=False)
    tail = np.arange(max(n - 2, 0), n)
    return np.unique(np.concatenate([txt, img, tail]))


def _check_rows(y, x, ref, rows, what):
    assert_close(y[rows], ref, what)
    assert_delta_close(y[rows] - x[rows], ref - x[rows], what + " (branch delta)")


@pytest.mark.parametrize("name", ["block_2k", "block_2k_dh128", "block_4k", "block_4k_dh128",
                                  "edit_4ref", "edit_4ref_dh128"])
def test_full_width_block_sampled_rows(name):
    from image_generation_b200 import h3dit as H

    w = synth.WORKLOADS[name]
    d = w.dims
    tw = synth.time_weights(d, w.seed)
    bw = synth.block_weights(d, w.seed)
    inp = synth.workload_inputs(w)
    cfg = H.make_config(d.hidden, d.heads, d.head_dim, d.ffn, 1, w.n_tokens, io_fp32=True)
    ctx = H.Context(cfg, time_tensors(tw), [block_tensors(bw)])
    xt, xi = to_dev(inp["x_txt"], "f32"), to_dev(inp["x_img"], "f32")
    ctx.block_forward(0, inp["t"], xi, list(w.grids), xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    y = np.concatenate([to_np(xt), to_np(xi)], axis=0)
    del ctx, xt, xi
    torch.cuda.empty_cache()

    ocfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
    x = O.pack(inp["x_txt"], inp["x_img"])
    mod = O.adaln_modulation(O.timestep_condition(inp["t"], tw, ocfg), bw["w_ada"], bw["b_ada"])
    rows = _sample_rows(w.n_txt, w.n_tokens, w.seed)
    ref = O.block_forward(x, mod, bw, O.token_positions(w.n_txt, w.grids), ocfg, rows=rows)
    _check_rows(y, x, ref, rows, name)


@pytest.mark.parametrize("live", [17])
def test_step_full_size_one_live_block(live):
    """h3dit_step over 50 blocks at the 4096^2 workload. Every block but one has
    zero gates (its AdaLN gate rows and bias are zero), which leaves the fp32
    residual exactly unchanged while all of its kernels still run; the step's
    output must then equal the live block alone, as the oracle computes it."""
    from image_generation_b200 import h3dit as H

    w = synth.WORKLOADS["block_4k"]
    d = w.dims
    D = d.hidden
    tw = synth.time_weights(d, w.seed)
    bw_live = synth.block_weights(d, 77)
    inp = synth.workload_inputs(w)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    blocks = []
    for l in range(synth.N_BLOCKS):
        if l == live:
            blocks.append(block_tensors(bw_live))
            continue
        I = d.inner
        rnd = lambda *s: (torch.randn(*s, device="cuda", generator=gen) * 0.02).bfloat16()
        wada = rnd(6 * D, D)
        wada[2 * D:3 * D] = 0   # gate1
        wada[5 * D:6 * D] = 0   # gate2
        blocks.append({"w_qkv": rnd(3 * I, D), "w_o": rnd(D, I), "w_ff1": rnd(d.ffn, D),
                       "w_ff2": rnd(D, d.ffn), "w_ada": wada,
                       "b_ada": torch.zeros(6 * D, device="cuda")})
    cfg = H.make_config(D, d.heads, d.head_dim, d.ffn, synth.N_BLOCKS, w.n_tokens, io_fp32=True)
    ctx = H.Context(cfg, time_tensors(tw), blocks)
    xt, xi = to_dev(inp["x_txt"], "f32"), to_dev(inp["x_img"], "f32")
    t = synth.step_timesteps()[1]
    ctx.step(t, xi, list(w.grids), xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    y = np.concatenate([to_np(xt), to_np(xi)], axis=0)
    del ctx, blocks, xt, xi
    torch.cuda.empty_cache()

    ocfg = O.config_for(D, d.heads, d.head_dim, d.ffn)
    x = O.pack(inp["x_txt"], inp["x_img"])
    mod = O.adaln_modulation(O.timestep_condition(t, tw, ocfg), bw_live["w_ada"], bw_live["b_ada"])
    rows = _sample_rows(w.n_txt, w.n_tokens, 9, k_img=96)
    ref = O.block_forward(x, mod, bw_live, O.token_positions(w.n_txt, w.grids), ocfg, rows=rows)
    _check_rows(y, x, ref, rows, "50-block step, one live block")


def test_step_full_size_zero_gates_is_identity():
    """With every gate zero the 50-block step returns its input bit for bit."""
    from image_generation_b200 import h3dit as H

    d = synth.FULL_96
    D, I = d.hidden, d.inner
    n_txt, grid = 512, 128
    gen = torch.Generator(device="cuda")
    gen.manual_seed(6)
    rnd = lambda *s: (torch.randn(*s, device="cuda", generator=gen) * 0.02).bfloat16()
    blocks = []
    for _ in range(synth.N_BLOCKS):
        wada = rnd(6 * D, D)
        wada[2 * D:3 * D] = 0
        wada[5 * D:6 * D] = 0
        blocks.append({"w_qkv": rnd(3 * I, D), "w_o": rnd(D, I), "w_ff1": rnd(d.ffn, D),
                       "w_ff2": rnd(D, d.ffn), "w_ada": wada, "b_ada": torch.zeros(6 * D, device="cuda")})
    tw = {k: to_dev(v, "f32") for k, v in synth.time_weights(d, 1).items()}
    cfg = H.make_config(D, d.heads, d.head_dim, d.ffn, synth.N_BLOCKS, n_txt + grid * grid)
    ctx = H.Context(cfg, tw, blocks)
    xt = torch.randn(n_txt, D, device="cuda", generator=gen).bfloat16()
    xi = torch.randn(grid * grid, D, device="cuda", generator=gen).bfloat16()
    xt0, xi0 = xt.clone(), xi.clone()
    ctx.step(0.5, xi, [(0, grid, grid)], xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    assert torch.equal(xt, xt0) and torch.equal(xi, xi0)
