"""Parity of the whole block and of the multi-block step, through the C ABI,
against the oracle; plus the GPU side of the boundary's argument checks."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import assert_close, assert_delta_close, block_tensors, time_tensors, to_dev, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ctx(dims, bws, tw, max_tokens, **kw):
    from image_generation_b200 import h3dit as H

    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, len(bws), max_tokens, **kw)
    return H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws])


def _run_block(ctx, block, t, x_txt, x_img, grids, mod=None):
    kind = "f32" if ctx.cfg.io_fp32 else "bf16"
    xt = to_dev(x_txt, kind) if x_txt.shape[0] else None
    xi = to_dev(x_img, kind)
    ctx.block_forward(block, t, xi, grids, xt, mod=None if mod is None else to_dev(mod, "f32"))
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    y_txt = to_np(xt) if xt is not None else np.zeros((0, x_img.shape[1]))
    return np.concatenate([y_txt, to_np(xi)], axis=0)


def _check_block(y, x, ref, what, delta=True):
    """The output, and with fp32 token buffers also the branch delta y - x
    (with bf16 buffers the output rounding alone would swamp a small delta)."""
    assert_close(y, ref, what)
    if delta:
        assert_delta_close(y - x, ref - x, what + " (branch delta)")


@pytest.mark.parametrize("io_fp32", [False, True])
@pytest.mark.parametrize("head_dim,gelu_tanh", [(96, False), (128, False), (96, True)])
def test_small_block_against_oracle(head_dim, gelu_tanh, io_fp32):
    w = synth.WORKLOADS["small_block"]
    dims = w.dims if head_dim == 96 else synth.Dims(768, 6, 128, 2048)
    tw = synth.time_weights(dims, w.seed)
    bw = synth.block_weights(dims, w.seed)
    inp = synth.workload_inputs(w)
    ctx = _ctx(dims, [bw], tw, w.n_tokens, gelu_tanh=gelu_tanh, io_fp32=io_fp32)
    y = _run_block(ctx, 0, inp["t"], inp["x_txt"], inp["x_img"], list(w.grids))
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn, gelu_tanh=gelu_tanh)
    x = O.pack(inp["x_txt"], inp["x_img"])
    mod = O.adaln_modulation(O.timestep_condition(inp["t"], tw, ocfg), bw["w_ada"], bw["b_ada"])
    ref = O.block_forward(x, mod, bw, O.token_positions(w.n_txt, w.grids), ocfg)
    _check_block(y, x, ref, f"small block d_h={head_dim}", delta=io_fp32)


@pytest.mark.parametrize("n_txt,grids", [(0, [(0, 9, 13)]), (5, [(0, 7, 7), (1, 3, 5), (2, 11, 2)]),
                                         (129, [(0, 1, 1)])])
def test_ragged_block_with_given_modulation(n_txt, grids):
    dims = synth.SMALL
    tw = synth.time_weights(dims, 3)
    bw = synth.block_weights(dims, 3)
    n_img = sum(h * w for _, h, w in grids)
    x_txt = synth.tokens(n_txt, dims.hidden, 3, "t")
    x_img = synth.tokens(n_img, dims.hidden, 3, "i")
    mod = synth.normal_f32((6, dims.hidden), 0.3, 3, "mod")
    ctx = _ctx(dims, [bw], tw, 512, io_fp32=True)
    y = _run_block(ctx, 0, 0.0, x_txt, x_img, grids, mod=mod)
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    x = O.pack(x_txt, x_img)
    ref = O.block_forward(x, mod, bw, O.token_positions(n_txt, grids), ocfg)
    _check_block(y, x, ref, f"ragged block n={x.shape[0]}")


def test_zero_gates_leave_tokens_bit_exact():
    dims = synth.SMALL
    bw = synth.block_weights(dims, 4)
    tw = synth.time_weights(dims, 4)
    mod = synth.normal_f32((6, dims.hidden), 0.3, 4, "mod")
    mod[2] = 0.0
    mod[5] = 0.0
    x_txt = synth.tokens(17, dims.hidden, 4, "t")
    x_img = synth.tokens(200, dims.hidden, 4, "i")
    ctx = _ctx(dims, [bw], tw, 512)
    y = _run_block(ctx, 0, 0.3, x_txt, x_img, [(0, 10, 20)], mod=mod)
    assert np.array_equal(y, O.pack(x_txt, x_img))


def test_text_permutation_equivariance_on_gpu():
    dims = synth.SMALL
    bw = synth.block_weights(dims, 6)
    tw = synth.time_weights(dims, 6)
    x_txt = synth.tokens(9, dims.hidden, 6, "t")
    x_img = synth.tokens(64, dims.hidden, 6, "i")
    ctx = _ctx(dims, [bw], tw, 128)
    y = _run_block(ctx, 0, 0.6, x_txt, x_img, [(0, 8, 8)])
    perm = np.array([4, 0, 8, 2, 6, 1, 3, 7, 5])
    yp = _run_block(ctx, 0, 0.6, x_txt[perm], x_img, [(0, 8, 8)])
    assert_close(yp[:9], y[perm], "permuted text rows")
    assert_close(yp[9:], y[9:], "image rows under text permutation")


def test_step_fifty_blocks_small_width():
    w = synth.WORKLOADS["small_block"]
    dims = w.dims
    tw = synth.time_weights(dims, w.seed)
    bws = [synth.block_weights(dims, 1000 + l) for l in range(synth.N_BLOCKS)]
    inp = synth.workload_inputs(w)
    ctx = _ctx(dims, bws, tw, w.n_tokens, io_fp32=True)
    xt, xi = to_dev(inp["x_txt"], "f32"), to_dev(inp["x_img"], "f32")
    t = synth.step_timesteps()[2]
    ctx.step(t, xi, list(w.grids), xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    y = np.concatenate([to_np(xt), to_np(xi)], axis=0)
    ocfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    x = O.pack(inp["x_txt"], inp["x_img"])
    ref = O.step_forward(x, t, tw, bws, O.token_positions(w.n_txt, w.grids), ocfg)
    _check_block(y, x, ref, "50-block step")


def test_step_is_run_to_run_deterministic():
    """No kernel of the step reduces through atomics or in an order that
    depends on scheduling: every output element is summed by one CTA in a
    fixed order. Two runs on the same inputs therefore agree bit for bit.
    Checked on a 50-block step over 2,116 tokens, which spans many GEMM and
    attention tiles with ragged tails."""
    dims = synth.SMALL
    tw = synth.time_weights(dims, 8)
    bws = [synth.block_weights(dims, 1100 + l) for l in range(synth.N_BLOCKS)]
    x_txt = synth.tokens(52, dims.hidden, 8, "t")
    x_img = synth.tokens(48 * 43, dims.hidden, 8, "i")
    ctx = _ctx(dims, bws, tw, 2200, io_fp32=True)
    outs = []
    for _ in range(2):
        xt, xi = to_dev(x_txt, "f32"), to_dev(x_img, "f32")
        ctx.step(0.7, xi, [(0, 48, 43)], xt)
        torch.cuda.synchronize()
        assert ctx.sync_status() == 0
        outs.append(np.concatenate([to_np(xt), to_np(xi)], axis=0))
    assert np.isfinite(outs[0]).all()
    assert np.array_equal(outs[0], outs[1])
    assert not np.array_equal(outs[0], O.pack(x_txt, x_img))  # the step did change the tokens


def test_boundary_errors_with_a_live_context():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    bw = synth.block_weights(dims, 1)
    tw = synth.time_weights(dims, 1)
    ctx = _ctx(dims, [bw], tw, 64)
    xi = torch.zeros(64, dims.hidden, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.H3DitError) as e:   # more tokens than max_tokens
        ctx.block_forward(0, 0.5, xi, [(0, 9, 9)], None)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    with pytest.raises(H.H3DitError) as e:   # block index out of range
        ctx.block_forward(1, 0.5, xi, [(0, 8, 8)], None)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    a = torch.zeros(8, 96, dtype=torch.bfloat16, device="cuda")
    wt = torch.zeros(64, 96, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.H3DitError) as e:   # k not a multiple of 64
        ctx.linear(H.H3DIT_EPI_STORE, a, wt, out)
    assert e.value.status == H.H3DIT_ERR_UNSUPPORTED
    with pytest.raises(H.H3DitError) as e:   # gated residual without a gate
        ctx.linear(H.H3DIT_EPI_GATED_RESIDUAL, a[:, :64].contiguous(), wt[:, :64].contiguous(),
                   out.float())
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    base = torch.zeros(1000, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.H3DitError) as e:   # misaligned attention operand
        ctx.attention(base[1:], base, base, 768, base, 768, 1)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    assert ctx.sync_status() == 0
