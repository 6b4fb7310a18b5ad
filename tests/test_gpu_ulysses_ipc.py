"""Ulysses with the fused exchanges across real processes: 2 and 4 ranks,
and 2 with the MXFP8 linears, each its own process and CUDA context on
cuda:0. They map one another's receive and output buffers (and, in MXFP8, the
output scales) with CUDA IPC (connect_peers: handles exchanged over gloo,
h3dit_ipc_open in every other process), run a 2-block step with the host
barrier after each fused stage (stream synchronise, then a gloo barrier), and
must reproduce the unsharded step bit for bit. This is the whole
multi-process path of the fused form - peer mapping, byte offsets inside the
caching allocator's segments, barriers, unmapping - with the peers on one
device. No kernel waits on another rank: every rank's kernels only store, and
the ordering comes from the host barrier."""
import datetime
import os
import socket

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _rank_main(rank, world, port, mx, out):
    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        from image_generation_b200 import h3dit as H
        from image_generation_b200 import synth
        from image_generation_b200.ulysses import UlyssesStep, host_barrier
        from tests.helpers import block_tensors, time_tensors

        dims, n_blocks, n_txt, grids = synth.SMALL, 2, 32, [(0, 16, 16)]
        n_total = n_txt + 256
        tw = time_tensors(synth.time_weights(dims, 1))
        weights = [block_tensors(synth.block_weights(dims, 101 + l)) for l in range(n_blocks)]
        cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, n_blocks, n_total,
                            io_fp32=True,
                            precision=H.H3DIT_PRECISION_MXFP8 if mx else H.H3DIT_PRECISION_BF16)
        ctx = H.Context(cfg, tw, weights)
        g = torch.Generator(device="cuda")
        g.manual_seed(1)
        x = torch.randn(n_total, dims.hidden, device="cuda", generator=g)
        barrier = host_barrier()
        step = UlyssesStep(ctx, weights, rank, world, n_total, dims.hidden, dims.heads,
                           dims.head_dim, dims.ffn, fused=True, barrier=barrier, mx=mx)
        own = step.r.recv_ptrs[rank] == step.r.recv.data_ptr()
        others = len({p for i, p in enumerate(step.r.recv_ptrs) if i != rank}) == world - 1
        xl = x[step.r.rows()].clone()
        step(0.4, xl, grids, n_txt)
        barrier()
        step.close()
        dist.barrier()
        st = ctx.sync_status()
        rows = [torch.empty(xl.shape, dtype=xl.dtype) for _ in range(world)]
        dist.all_gather(rows, xl.cpu())
        if rank == 0:
            xt, xi = x[:n_txt].clone(), x[n_txt:].clone()
            ctx.step(0.4, xi, grids, xt)
            torch.cuda.synchronize()
            ref = torch.cat([xt, xi]).cpu()
            got = torch.cat(rows)
            out.update(equal=bool(torch.equal(got, ref)),
                       maxdiff=float((got - ref).abs().max()),
                       changed=not torch.equal(ref, x.cpu()),
                       status=st + ctx.sync_status(), own=own, others=others)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,mx", [(2, False), (4, False), (2, True)],
                         ids=["sp2", "sp4", "sp2_mxfp8"])
def test_fused_exchange_across_processes_with_ipc(world, mx):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, mx, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=600)
        for p in procs:
            if p.is_alive():
                p.terminate()
                p.join(timeout=30)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert all(c == 0 for c in codes), codes
    assert res["status"] == 0
    assert res["own"] and res["others"]
    assert res["changed"]
    assert res["equal"], f"max diff {res['maxdiff']}"
