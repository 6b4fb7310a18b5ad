"""Runtime behaviour on the GPU: a bounded wait that runs out is reported
through the status word without faulting anything, kernels started while it
is set do no work, and the context works again once it is read; a step
captured in a CUDA graph replays bit for bit like eager launches (the
graph-versus-eager agreement check the vLLM post describes for its decoder)."""
import numpy as np
import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import assert_bf16_rounding, block_tensors, time_tensors, to_dev, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ctx(dims, n_blocks, max_tokens, seed=0, **kw):
    from image_generation_b200 import h3dit as H

    tw = synth.time_weights(dims, seed)
    bws = [synth.block_weights(dims, seed + 1000 + l) for l in range(n_blocks)]
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, max_tokens, **kw)
    return H.Context(cfg, time_tensors(tw), [block_tensors(b) for b in bws])


def test_bounded_wait_times_out_and_the_context_recovers():
    from image_generation_b200 import h3dit as H

    ctx = _ctx(synth.SMALL, 1, 64)
    a = synth.tokens(130, 768, 1, "a")
    w = synth.normal_bf16((256, 768), 0.02, 1, "w")
    ad, wd = to_dev(a), to_dev(w)
    out = torch.full((130, 256), 7.0, dtype=torch.bfloat16, device="cuda")

    ctx.selftest_bounded_wait(20000)         # 20 ms wait on a barrier nothing arrives on
    ctx.linear(H.H3DIT_EPI_STORE, ad, wd, out)  # started while the status is set: no work
    torch.cuda.synchronize()
    assert ctx.sync_status() == H.H3DIT_ERR_TIMEOUT
    assert bool((out == 7.0).all())
    assert ctx.sync_status() == H.H3DIT_OK     # read once, then cleared

    ctx.linear(H.H3DIT_EPI_STORE, ad, wd, out)
    torch.cuda.synchronize()
    assert ctx.sync_status() == H.H3DIT_OK
    assert_bf16_rounding(to_np(out), O.linear(a, w), "linear after recovery", abs_floor=1e-3)


def test_graph_captured_step_equals_eager_bit_for_bit():
    w = synth.WORKLOADS["small_block"]
    ctx = _ctx(w.dims, 4, w.n_tokens)
    inp = synth.workload_inputs(w)
    grids = list(w.grids)
    t = 0.75

    xt_e, xi_e = to_dev(inp["x_txt"]), to_dev(inp["x_img"])
    ctx.step(t, xi_e, grids, xt_e)                  # eager (also warms every kernel up)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0

    xt_g, xi_g = to_dev(inp["x_txt"]), to_dev(inp["x_img"])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ctx.step(t, xi_g, grids, xt_g)
    for _ in range(2):                               # replay twice from fresh inputs
        xt_g.copy_(to_dev(inp["x_txt"]))
        xi_g.copy_(to_dev(inp["x_img"]))
        graph.replay()
        torch.cuda.synchronize()
        assert ctx.sync_status() == 0
        assert torch.equal(xt_g, xt_e) and torch.equal(xi_g, xi_e)
    del graph
