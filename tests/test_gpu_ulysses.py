"""Ulysses sequence parallelism on the GPU path, with P ranks emulated in one
process on one GPU: each rank's stages run libh3dit's kernels through
image_generation_b200.ulysses (RMSNorm, QKV + RoPE on its rows, the head-group
re-layouts, attention on its head group, out-projection and FFN), and the two
all-to-alls are done by device copies between the ranks' buffers - the same
data movement NCCL's all_to_all_single does between GPUs. No kernel waits on
another rank. Every kernel computes each output element the same way whatever
rows or heads it is given, so the result must equal the unsharded step bit
for bit."""
import pytest

from image_generation_b200 import synth
from tests.helpers import block_tensors, time_tensors

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _exchange_qkv(ranks):
    P = len(ranks)
    for d in range(P):
        for s in range(P):
            ranks[d].recv1[s].copy_(ranks[s].send1[d])


def _exchange_o(ranks):
    P = len(ranks)
    n = ranks[0].n
    for d in range(P):
        for s in range(P):
            ranks[d].recv2[s].copy_(ranks[s].o_heads[d * n:(d + 1) * n])


def _emulated_step(ctx, weights, P, dims, t, x, grids, n_txt):
    from image_generation_b200.ulysses import UlyssesRank

    n_total = x.shape[0]
    ranks = [UlyssesRank(ctx, r, P, n_total, dims.hidden, dims.heads, dims.head_dim, dims.ffn)
             for r in range(P)]
    c = torch.empty(dims.hidden, device="cuda")
    mod = torch.empty(len(weights), 6, dims.hidden, device="cuda")
    rope = torch.empty(n_total, dims.head_dim // 2, 2, device="cuda")
    ctx.time_embed(t, c)
    ctx.adaln_project(c, 0, len(weights), mod)
    ctx.rope_table(grids, n_txt, rope)
    xs = [x[r.rows()].clone() for r in ranks]
    for l, w in enumerate(weights):
        for i, r in enumerate(ranks):
            r.qkv_and_pack(xs[i], mod[l], w, rope[r.rows()])
        _exchange_qkv(ranks)
        for r in ranks:
            r.attention()
        _exchange_o(ranks)
        for i, r in enumerate(ranks):
            r.finish(xs[i], mod[l], w)
    return torch.cat(xs)


def _run(dims, n_blocks, P, n_txt, grids, seed):
    from image_generation_b200 import h3dit as H

    tw = time_tensors(synth.time_weights(dims, seed))
    weights = [block_tensors(synth.block_weights(dims, seed + 100 + l)) for l in range(n_blocks)]
    n_total = n_txt + sum(h * w for _, h, w in grids)
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, n_total,
                        io_fp32=True)
    ctx = H.Context(cfg, tw, weights)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn(n_total, dims.hidden, device="cuda", generator=g)
    got = _emulated_step(ctx, weights, P, dims, 0.4, x, grids, n_txt)
    xt, xi = x[:n_txt].clone(), x[n_txt:].clone()
    ctx.step(0.4, xi, grids, xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    ref = torch.cat([xt, xi])
    assert not torch.equal(ref, x)
    return got, ref


@pytest.mark.parametrize("P", [2, 4, 8])
def test_emulated_ranks_small(P):
    got, ref = _run(synth.SMALL, 2, P, 32, [(0, 16, 16)], 1)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def test_emulated_ranks_head_dim_128():
    dims = synth.Dims(hidden=768, heads=8, head_dim=128, ffn=2048)
    got, ref = _run(dims, 2, 4, 8, [(0, 12, 20), (1, 4, 4)], 2)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


@pytest.mark.parametrize("P", [4, 8])
def test_emulated_ranks_full_width_4096(P):
    """SP4 and SP8 at full width on the 4096^2 sequence (16,896 tokens, 14 and 7
    heads per rank), one block."""
    got, ref = _run(synth.FULL_96, 1, P, 512, [(0, 128, 128)], 3)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def _emulated_step_fused(ctx, weights, P, dims, t, x, grids, n_txt):
    """The fused form: each rank's QKV GEMM and attention write straight into
    the other ranks' buffers (here all on one GPU, so stream order stands in
    for the barrier between the stages)."""
    from image_generation_b200.ulysses import FusedUlyssesRank, fused_block

    n_total = x.shape[0]
    ranks = [FusedUlyssesRank(ctx, r, P, n_total, dims.hidden, dims.heads, dims.head_dim,
                              dims.ffn) for r in range(P)]
    recv_ptrs = [r.recv.data_ptr() for r in ranks]
    o_ptrs = [r.o.data_ptr() for r in ranks]
    for r in ranks:
        r.recv.fill_(float("nan"))
        r.o.fill_(float("nan"))
        r.connect(recv_ptrs, o_ptrs)
    c = torch.empty(dims.hidden, device="cuda")
    mod = torch.empty(len(weights), 6, dims.hidden, device="cuda")
    rope = torch.empty(n_total, dims.head_dim // 2, 2, device="cuda")
    ctx.time_embed(t, c)
    ctx.adaln_project(c, 0, len(weights), mod)
    ctx.rope_table(grids, n_txt, rope)
    xs = [x[r.rows()].clone() for r in ranks]
    for l, w in enumerate(weights):
        for i, r in enumerate(ranks):
            r.qkv_scatter(xs[i], mod[l], w, rope[r.rows()])
        for r in ranks:
            r.attention_scatter()
        for i, r in enumerate(ranks):
            r.finish(xs[i], mod[l], w)
    return torch.cat(xs)


def _run_fused(dims, n_blocks, P, n_txt, grids, seed):
    from image_generation_b200 import h3dit as H

    tw = time_tensors(synth.time_weights(dims, seed))
    weights = [block_tensors(synth.block_weights(dims, seed + 100 + l)) for l in range(n_blocks)]
    n_total = n_txt + sum(h * w for _, h, w in grids)
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, n_total,
                        io_fp32=True)
    ctx = H.Context(cfg, tw, weights)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn(n_total, dims.hidden, device="cuda", generator=g)
    got = _emulated_step_fused(ctx, weights, P, dims, 0.4, x, grids, n_txt)
    xt, xi = x[:n_txt].clone(), x[n_txt:].clone()
    ctx.step(0.4, xi, grids, xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    ref = torch.cat([xt, xi])
    assert not torch.equal(ref, x)
    return got, ref


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_fused_exchange_emulated_ranks_small(P):
    got, ref = _run_fused(synth.SMALL, 2, P, 32, [(0, 16, 16)], 1)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def test_fused_exchange_head_dim_128_ragged_tiles():
    """d_h 128 (rotary units of 32 and 48 columns) on 4 x 300 = 1,200 tokens:
    each rank's 300 rows end inside a 256-row GEMM tile, and the attention's
    last query and key tiles run past the sequence."""
    dims = synth.Dims(hidden=768, heads=8, head_dim=128, ffn=2048)
    got, ref = _run_fused(dims, 2, 4, 8, [(0, 32, 37), (1, 4, 2)], 2)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


@pytest.mark.parametrize("P", [4, 8])
def test_fused_exchange_full_width_4096(P):
    """SP4 and SP8 at full width on the 4096^2 sequence, one block."""
    got, ref = _run_fused(synth.FULL_96, 1, P, 512, [(0, 128, 128)], 3)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def _run_fused_mx(dims, n_blocks, P, n_txt, grids, seed):
    """The fused exchanges on an MXFP8 context: each rank quantizes its rows,
    its QKV (the context's quantized weights) stores into every rank's bf16
    receive buffer, and its attention writes MXFP8 rows and scales into every
    rank's out-projection input; compared with the unsharded MXFP8 step."""
    from image_generation_b200 import h3dit as H
    from image_generation_b200.ulysses import FusedUlyssesRank

    tw = time_tensors(synth.time_weights(dims, seed))
    weights = [block_tensors(synth.block_weights(dims, seed + 100 + l)) for l in range(n_blocks)]
    n_total = n_txt + sum(h * w for _, h, w in grids)
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, n_total,
                        io_fp32=True, precision=H.H3DIT_PRECISION_MXFP8)
    ctx = H.Context(cfg, tw, weights)
    ranks = [FusedUlyssesRank(ctx, r, P, n_total, dims.hidden, dims.heads, dims.head_dim,
                              dims.ffn, mx=True) for r in range(P)]
    for r in ranks:
        r.recv.fill_(float("nan"))
        r.connect([q.recv.data_ptr() for q in ranks], [q.o.data_ptr() for q in ranks],
                  [q.o_sf.data_ptr() for q in ranks])
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn(n_total, dims.hidden, device="cuda", generator=g)
    c = torch.empty(dims.hidden, device="cuda")
    mod = torch.empty(n_blocks, 6, dims.hidden, device="cuda")
    rope = torch.empty(n_total, dims.head_dim // 2, 2, device="cuda")
    ctx.time_embed(0.4, c)
    ctx.adaln_project(c, 0, n_blocks, mod)
    ctx.rope_table(grids, n_txt, rope)
    xs = [x[r.rows()].clone() for r in ranks]
    for l, w in enumerate(weights):
        for i, r in enumerate(ranks):
            r.qkv_scatter(xs[i], mod[l], w, rope[r.rows()], block=l)
        for r in ranks:
            r.attention_scatter()
        for i, r in enumerate(ranks):
            r.finish(xs[i], mod[l], w, block=l)
    got = torch.cat(xs)
    xt, xi = x[:n_txt].clone(), x[n_txt:].clone()
    ctx.step(0.4, xi, grids, xt)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    ref = torch.cat([xt, xi])
    assert not torch.equal(ref, x)
    return got, ref


@pytest.mark.parametrize("P", [2, 4, 8])
def test_fused_exchange_mxfp8_emulated_ranks_small(P):
    got, ref = _run_fused_mx(synth.SMALL, 2, P, 32, [(0, 16, 16)], 4)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def test_fused_exchange_mxfp8_head_dim_128_ragged():
    dims = synth.Dims(hidden=768, heads=8, head_dim=128, ffn=2048)
    got, ref = _run_fused_mx(dims, 2, 4, 8, [(0, 32, 37), (1, 4, 2)], 5)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def test_fused_exchange_mxfp8_full_width_4096():
    """SP4 with the MXFP8 linears at full width on the 4096^2 sequence, one
    block: the pages' latency configuration."""
    got, ref = _run_fused_mx(synth.FULL_96, 1, 4, 512, [(0, 128, 128)], 6)
    assert torch.equal(got, ref), f"max diff {float((got - ref).abs().max())}"


def test_fused_exchange_writes_only_its_blocks():
    """Every receive and output buffer sits between guard margins; the two
    fused calls of all ranks must fill the buffers and leave the margins."""
    from image_generation_b200 import h3dit as H
    from tests.test_gpu_guards import Guarded

    dims, P, n_txt, grids = synth.SMALL, 4, 4, [(0, 10, 10)]
    n_total = n_txt + 100
    n = n_total // P
    cw = dims.inner // P
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 1, n_total)
    bw = block_tensors(synth.block_weights(dims, 5))
    ctx = H.Context(cfg, time_tensors(synth.time_weights(dims, 5)), [bw])
    recv = [Guarded((n_total, 3 * cw), torch.bfloat16) for _ in range(P)]
    outs = [Guarded((n, dims.inner), torch.bfloat16) for _ in range(P)]
    rope = torch.empty(n_total, dims.head_dim // 2, 2, device="cuda")
    ctx.rope_table(grids, n_txt, rope)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    xm = (torch.randn(n_total, dims.hidden, device="cuda", generator=g)).bfloat16()
    for r in range(P):
        ctx.sp_qkv_scatter(xm[r * n:(r + 1) * n], bw["w_qkv"], rope[r * n:(r + 1) * n],
                           [b.t.data_ptr() for b in recv], r)
    for r in range(P):
        ctx.sp_attention_scatter(recv[r].t, [b.t.data_ptr() for b in outs], r)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    for i, b in enumerate(recv + outs):
        b.check(f"buffer {i}")
        assert not bool(torch.isnan(b.t.float()).any())


def test_fused_exchange_mxfp8_writes_only_its_blocks():
    """The MXFP8 form's stores (bf16 Q|K|V into the receive buffers, E4M3
    rows and their scales into the owners' out-projection inputs) stay inside
    each buffer and fill it: every buffer sits between guard margins. The
    300-row blocks of each rank end inside a 128-row block of the scale
    layout."""
    from image_generation_b200 import h3dit as H
    from tests.test_gpu_guards import Guarded

    dims, P, n = synth.SMALL, 4, 300
    n_total = P * n
    cw, I, D = dims.inner // P, dims.inner, dims.hidden
    cfg = H.make_config(D, dims.heads, dims.head_dim, dims.ffn, 1, n_total,
                        precision=H.H3DIT_PRECISION_MXFP8)
    bw = block_tensors(synth.block_weights(dims, 9))
    ctx = H.Context(cfg, time_tensors(synth.time_weights(dims, 9)), [bw])
    recv = [Guarded((n_total, 3 * cw), torch.bfloat16) for _ in range(P)]
    o = [Guarded((n, I), torch.uint8) for _ in range(P)]
    o_sf = [Guarded((H.mx_scale_bytes(n, I),), torch.uint8) for _ in range(P)]
    rope = torch.empty(n_total, dims.head_dim // 2, 2, device="cuda")
    ctx.rope_table([(0, 30, 40)], 0, rope)
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    x = torch.randn(n_total, D, device="cuda", generator=g)
    sh = torch.zeros(D, device="cuda")
    for r in range(P):
        xq = torch.empty(n, D, dtype=torch.uint8, device="cuda")
        xq_sf = torch.empty(H.mx_scale_bytes(n, D), dtype=torch.uint8, device="cuda")
        ctx.rmsnorm_modulate_mx(x[r * n:(r + 1) * n].contiguous(), sh, sh, xq, xq_sf)
        ctx.sp_qkv_scatter_mx(xq, xq_sf, 0, rope[r * n:(r + 1) * n],
                              [b.t.data_ptr() for b in recv], r)
    for r in range(P):
        ctx.sp_attention_scatter_mx(recv[r].t, [b.t.data_ptr() for b in o],
                                    [b.t.data_ptr() for b in o_sf], r)
    torch.cuda.synchronize()
    assert ctx.sync_status() == 0
    for i, b in enumerate(recv):
        b.check(f"receive buffer {i}")
        assert not bool(torch.isnan(b.t.float()).any())
    for i, (b, f) in enumerate(zip(o, o_sf)):
        b.check(f"E4M3 output {i}")
        f.check(f"scales {i}")
        # every code written (0xFF, the fill, is an E4M3 NaN the saturating
        # quantization never produces); the scale array's padding rows stay
        assert not bool((b.t == 0xFF).any()), f"E4M3 output {i} not filled"


def test_fused_exchange_errors():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 1, 64)
    bw = block_tensors(synth.block_weights(dims, 0))
    ctx = H.Context(cfg, time_tensors(synth.time_weights(dims, 0)), [bw])
    xm = torch.zeros(16, dims.hidden, device="cuda", dtype=torch.bfloat16)
    rope = torch.zeros(16, dims.head_dim // 2, 2, device="cuda")
    buf = torch.zeros(64, 3 * dims.inner, device="cuda", dtype=torch.bfloat16)
    p = buf.data_ptr()
    cases = [
        (lambda: ctx.sp_qkv_scatter(xm, bw["w_qkv"], rope, [p, p, p], 0), H.H3DIT_ERR_UNSUPPORTED),
        (lambda: ctx.sp_qkv_scatter(xm, bw["w_qkv"], rope, [p] * 16, 0), H.H3DIT_ERR_UNSUPPORTED),
        (lambda: ctx.sp_qkv_scatter(xm, bw["w_qkv"], rope, [p, p], 2), H.H3DIT_ERR_INVALID_ARG),
        (lambda: ctx.sp_qkv_scatter(xm, bw["w_qkv"], rope, [p, p + 2], 0), H.H3DIT_ERR_INVALID_ARG),
        (lambda: ctx.sp_qkv_scatter(xm, bw["w_qkv"], rope, [p, 0], 0), H.H3DIT_ERR_INVALID_ARG),
        (lambda: ctx.sp_attention_scatter(buf[:63], [p, p], 0), H.H3DIT_ERR_UNSUPPORTED),
    ]
    for call, status in cases:
        with pytest.raises(H.H3DitError) as e:
            call()
        assert e.value.status == status
    assert ctx.sync_status() == 0


def test_relayout_errors():
    from image_generation_b200 import h3dit as H

    dims = synth.SMALL
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 1, 64)
    ctx = H.Context(cfg, time_tensors(synth.time_weights(dims, 0)),
                    [block_tensors(synth.block_weights(dims, 0))])
    qkv = torch.zeros(16, 3 * dims.inner, device="cuda", dtype=torch.bfloat16)
    send = torch.zeros(3, 16, dims.inner, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(H.H3DitError) as e:   # 3 ranks do not divide 8 heads
        ctx.sp_pack_qkv(qkv, 3, send)
    assert e.value.status == H.H3DIT_ERR_UNSUPPORTED
    with pytest.raises(H.H3DitError) as e:   # more heads than the context has
        ctx.attention_heads(9, qkv, qkv, qkv, 3 * dims.inner, send.view(16, -1), 3 * dims.inner, 16)
    assert e.value.status == H.H3DIT_ERR_INVALID_ARG
    assert ctx.sync_status() == 0
