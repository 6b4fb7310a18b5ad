"""Layerwise weight streaming ("H3-Image Day-0 Support: 4K in 0.87s with Vera
Rubin", "Fitting Smaller GPUs"): blocks whose weights sit in pinned host
memory are copied into two alternating device staging slots while the
previous block computes. The kernels and their inputs are the same as with
resident weights, so every output must be bit-identical to the resident
context's - for any pattern of host and device blocks, for the step, a
single block and the whole denoise loop, eager or replayed from a CUDA graph."""
import numpy as np
import pytest

from image_generation_b200 import synth
from tests.helpers import block_tensors, time_tensors, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _weights(dims, n_blocks, seed=0):
    tw = time_tensors(synth.time_weights(dims, seed))
    bws = [block_tensors(synth.block_weights(dims, seed + 1000 + l)) for l in range(n_blocks)]
    return tw, bws


def _host(block):
    return {k: v.cpu().pin_memory() for k, v in block.items()}


def _pair(dims, n_blocks, host_blocks, max_tokens=300, io_fp32=False):
    """A resident context and one with `host_blocks` in pinned host memory."""
    from image_generation_b200 import h3dit as H

    tw, bws = _weights(dims, n_blocks)
    cfg = lambda: H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks,
                                max_tokens, io_fp32=io_fp32)
    ref = H.Context(cfg(), tw, bws)
    mixed = [(_host(b) if l in host_blocks else b) for l, b in enumerate(bws)]
    ctx = H.Context(cfg(), tw, mixed)
    assert ctx.streamed_blocks() == len(host_blocks)
    ctx.attach_staging()
    return ref, ctx


def _tokens(D, n_txt, n_img, seed, dt=torch.bfloat16):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return (torch.randn(n_txt, D, device="cuda", generator=g).to(dt),
            torch.randn(n_img, D, device="cuda", generator=g).to(dt))


@pytest.mark.parametrize("host_blocks", [(0, 1, 2, 3), (1, 3), (2, 3), (0,)],
                         ids=["all", "alternate", "tail", "first"])
def test_streamed_step_is_bit_identical(host_blocks):
    dims = synth.SMALL
    ref, ctx = _pair(dims, 4, set(host_blocks))
    grids = [(0, 16, 16)]
    xt, xi = _tokens(dims.hidden, 32, 256, 1)
    a_t, a_i, b_t, b_i = xt.clone(), xi.clone(), xt.clone(), xi.clone()
    for t in (1.0, 0.5):   # two steps: the slots are reused across calls
        ref.step(t, a_i, grids, a_t)
        ctx.step(t, b_i, grids, b_t)
    torch.cuda.synchronize()
    assert ref.sync_status() == 0 and ctx.sync_status() == 0
    assert torch.equal(a_t, b_t) and torch.equal(a_i, b_i)
    assert not torch.equal(a_i, xi)


def test_streamed_block_forward_and_given_modulation():
    dims = synth.SMALL
    D = dims.hidden
    ref, ctx = _pair(dims, 3, {1, 2})
    grids = [(0, 5, 7), (1, 3, 4)]
    xt, xi = _tokens(D, 3, 47, 2)
    for block in (0, 1, 2):
        a_t, a_i, b_t, b_i = xt.clone(), xi.clone(), xt.clone(), xi.clone()
        ref.block_forward(block, 0.3, a_i, grids, a_t)
        ctx.block_forward(block, 0.3, b_i, grids, b_t)
        torch.cuda.synchronize()
        assert torch.equal(a_t, b_t) and torch.equal(a_i, b_i), f"block {block}"
    mod = torch.randn(6, D, device="cuda") * 0.1
    a_t, a_i, b_t, b_i = xt.clone(), xi.clone(), xt.clone(), xi.clone()
    ref.block_forward(2, 0.0, a_i, grids, a_t, mod=mod)
    ctx.block_forward(2, 0.0, b_i, grids, b_t, mod=mod)
    torch.cuda.synchronize()
    assert ref.sync_status() == 0 and ctx.sync_status() == 0
    assert torch.equal(a_t, b_t) and torch.equal(a_i, b_i)


def test_streamed_denoise_is_bit_identical():
    dims = synth.SMALL
    D = dims.hidden
    ref, ctx = _pair(dims, 3, {0, 2}, io_fp32=True)
    f = lambda s, tag: torch.from_numpy(synth.normal_f32(s, 0.05, 8, tag)).cuda()
    io = {"w_in": f((D, 96), "w_in"), "b_in": f((D,), "b_in"), "w_mod": f((2 * D, D), "w_mod"),
          "b_mod": f((2 * D,), "b_mod"), "w_out": f((96, D), "w_out"), "b_out": f((96,), "b_out")}
    z = torch.randn(24, 32, 32, device="cuda")
    txt = torch.randn(32, D, device="cuda")
    za, zb = z.clone(), z.clone()
    ref.denoise(io, za, txt, 3)
    ctx.denoise(io, zb, txt, 3)
    torch.cuda.synchronize()
    assert ref.sync_status() == 0 and ctx.sync_status() == 0
    assert torch.equal(za, zb)


def test_streamed_step_in_a_cuda_graph():
    dims = synth.SMALL
    ref, ctx = _pair(dims, 4, {1, 2, 3})
    grids = [(0, 16, 16)]
    xt, xi = _tokens(dims.hidden, 32, 256, 3)
    b_t, b_i = xt.clone(), xi.clone()
    ctx.step(0.5, b_i, grids, b_t)   # untimed first call (per-device set-up)
    b_t.copy_(xt)
    b_i.copy_(xi)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        ctx.step(0.5, b_i, grids, b_t, stream=s)
    for _ in range(2):
        b_t.copy_(xt)
        b_i.copy_(xi)
        graph.replay()
    a_t, a_i = xt.clone(), xi.clone()
    ref.step(0.5, a_i, grids, a_t)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    assert torch.equal(a_t, b_t) and torch.equal(a_i, b_i)


def test_full_width_streamed_blocks_at_4096():
    """Full width at the 4096^2 canvas: 3 blocks, the last two in host memory
    (copied while the first computes), bit-identical to resident weights."""
    dims = synth.FULL_96
    ref, ctx = _pair(dims, 3, {1, 2}, max_tokens=16896)
    grids = [(0, 128, 128)]
    xt, xi = _tokens(dims.hidden, 512, 16384, 4)
    a_t, a_i, b_t, b_i = xt.clone(), xi.clone(), xt.clone(), xi.clone()
    ref.step(0.25, a_i, grids, a_t)
    ctx.step(0.25, b_i, grids, b_t)
    torch.cuda.synchronize()
    assert ref.sync_status() == 0 and ctx.sync_status() == 0
    assert torch.equal(a_t, b_t) and torch.equal(a_i, b_i)


def test_streaming_errors():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    tw, bws = _weights(dims, 2)
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 2, 300)
    ctx = H.Context(cfg, tw, [bws[0], _host(bws[1])])
    xt, xi = _tokens(dims.hidden, 32, 256, 5)
    with pytest.raises(H.H3DitError) as e:       # a host block and no staging
        ctx.step(0.5, xi, [(0, 16, 16)], xt)
    assert e.value.status == H.H3DIT_ERR_WORKSPACE
    ctx.block_forward(0, 0.5, xi, [(0, 16, 16)], xt)   # a resident block runs without it
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    with pytest.raises(H.H3DitError) as e:
        ctx.attach_staging(torch.empty(1024, dtype=torch.uint8, device="cuda"))
    assert e.value.status == H.H3DIT_ERR_WORKSPACE
    # one block split between host and device memory
    mixed = dict(bws[1])
    mixed["w_o"] = mixed["w_o"].cpu().pin_memory()
    with pytest.raises(H.H3DitError) as e:
        H.Context(cfg, tw, [bws[0], mixed])
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    # MXFP8 quantizes every block at create: host blocks are not run there
    mx = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 2, 300,
                       precision=H.H3DIT_PRECISION_MXFP8)
    with pytest.raises(H.H3DitError) as e:
        H.Context(mx, tw, [bws[0], _host(bws[1])])
    assert e.value.status == H.H3DIT_ERR_UNSUPPORTED
