"""Ulysses sequence parallelism ("H3-Image Day-0 Support: 4K in 0.87s with
Vera Rubin", "Faster DiT": Ulysses SP4) checked on the CPU with real gloo
ranks: every rank runs image_generation_b200.ulysses on its slice of the
packed sequence, with the two all-to-alls done by torch.distributed over
gloo and every step of the block done by the float64 oracle (an `ops` object
with the binding's method names). The rows gathered from all ranks must equal
the unsharded oracle step to float64 rounding: the partition, the RoPE rows
of each slice, the head-group re-layouts and both exchanges are then right.
The same driver runs on the GPU with libh3dit's kernels as `ops` and NCCL as
the exchange (tests/test_gpu_ulysses.py emulates the ranks on one GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from image_generation_b200 import synth
from oracle import dit_block as O

EPI_STORE, EPI_QKV_ROPE, EPI_GELU, EPI_GATED = 0, 1, 2, 3


def rotate_with_table(x, table, sections):
    """RoPE from a (cos, sin) table [n, d/2, 2] with the pairs ordered frame,
    row, col axis: axis a owns channels [o_a, o_a + 2 s_a), pair j is
    (o_a + j, o_a + s_a + j). x [n, H, d]."""
    out = x.copy()
    o = p = 0
    for s in sections:
        cos = table[:, None, p:p + s, 0]
        sin = table[:, None, p:p + s, 1]
        x1, x2 = x[..., o:o + s], x[..., o + s:o + 2 * s]
        out[..., o:o + s] = x1 * cos - x2 * sin
        out[..., o + s:o + 2 * s] = x2 * cos + x1 * sin
        o += 2 * s
        p += s
    return out


class OracleOps:
    """The binding's method names over the float64 oracle (CPU tensors)."""

    def __init__(self, cfg: O.BlockConfig, tw, bws):
        self.cfg, self.tw, self.bws = cfg, tw, bws

    def empty(self, shape, kind):
        return torch.full(tuple(shape), float("nan"), dtype=torch.float64)

    def time_embed(self, t, c):
        c[:] = torch.from_numpy(O.timestep_condition(t, self.tw, self.cfg))

    def adaln_project(self, c, first, count, mod):
        for i in range(count):
            b = self.bws[first + i]
            mod[i] = torch.from_numpy(O.adaln_modulation(c.numpy(), b["w_ada"], b["b_ada"]))

    def rope_table(self, grids, n_txt, table):
        ang = O.rope_angles(O.token_positions(n_txt, grids), self.cfg.rope_sections,
                            self.cfg.rope_theta)
        table[..., 0] = torch.from_numpy(np.cos(ang))
        table[..., 1] = torch.from_numpy(np.sin(ang))

    def rmsnorm_modulate(self, x, shift, scale, out):
        out[:] = torch.from_numpy(O.norm_modulate(x.numpy(), shift.numpy(), scale.numpy(),
                                                  self.cfg.norm_eps))

    def linear(self, epi, a, w, out, gate=None, rope_table=None):
        y = O.linear(a.numpy(), w)
        if epi == EPI_GELU:
            y = O.gelu(y)
        if epi == EPI_QKV_ROPE:
            n, I, c = y.shape[0], self.cfg.inner, self.cfg
            tab = rope_table.numpy()
            q = rotate_with_table(y[:, :I].reshape(n, c.heads, c.head_dim), tab, c.rope_sections)
            k = rotate_with_table(y[:, I:2 * I].reshape(n, c.heads, c.head_dim), tab,
                                  c.rope_sections)
            y = np.concatenate([q.reshape(n, I), k.reshape(n, I), y[:, 2 * I:]], axis=1)
        if epi == EPI_GATED:
            out += torch.from_numpy(gate.numpy() * y)
        else:
            out[:] = torch.from_numpy(y)

    def sp_pack_qkv(self, qkv, ranks, send):
        I = self.cfg.inner
        cw = I // ranks
        for d in range(ranks):
            cols = [slice(m * I + d * cw, m * I + (d + 1) * cw) for m in range(3)]
            send[d] = torch.cat([qkv[:, c] for c in cols], dim=1)

    def attention_heads(self, heads, q, k, v, ld_qkv, o, ld_o, n):
        d = self.cfg.head_dim
        w = heads * d
        r = lambda t: t[:, :w].numpy().reshape(n, heads, d)
        o[:, :w] = torch.from_numpy(O.attention(r(q), r(k), r(v)).reshape(n, w))

    def sp_unpack_o(self, recv, ranks, o):
        cw = self.cfg.inner // ranks
        for s in range(ranks):
            o[:, s * cw:(s + 1) * cw] = recv[s]


def _case(head_dim, n_blocks=2):
    dims = (synth.SMALL if head_dim == 96
            else synth.Dims(hidden=768, heads=8, head_dim=128, ffn=2048))
    cfg = O.config_for(dims.hidden, dims.heads, dims.head_dim, dims.ffn)
    tw = synth.time_weights(dims, 3)
    bws = [synth.block_weights(dims, 300 + l) for l in range(n_blocks)]
    n_txt, grids = 32, [(0, 16, 16)]
    x = O.pack(synth.tokens(n_txt, dims.hidden, 3, "txt"),
               synth.tokens(256, dims.hidden, 3, "img"))
    return dims, cfg, tw, bws, n_txt, grids, x


def _rank_main(rank, world, port, head_dim, out):
    import torch.distributed as dist

    from image_generation_b200.ulysses import UlyssesStep

    torch.set_num_threads(2)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dims, cfg, tw, bws, n_txt, grids, x = _case(head_dim)
        ops = OracleOps(cfg, tw, bws)
        weights = [{k: v for k, v in b.items()} for b in bws]
        n_total = x.shape[0]
        step = UlyssesStep(ops, weights, rank, world, n_total, dims.hidden, dims.heads,
                           dims.head_dim, dims.ffn)
        xl = torch.from_numpy(x[step.r.rows()].copy())
        step(0.6, xl, grids, n_txt)
        rows = [torch.empty_like(xl) for _ in range(world)]
        dist.all_gather(rows, xl)
        if rank == 0:
            out["y"] = torch.cat(rows).numpy()
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,head_dim", [(2, 96), (4, 96), (2, 128), (8, 128)],
                         ids=["sp2", "sp4", "sp2_dh128", "sp8_dh128"])
def test_ulysses_ranks_match_the_unsharded_step(world, head_dim):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, head_dim, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        y = out["y"]
    dims, cfg, tw, bws, n_txt, grids, x = _case(head_dim)
    ref = O.step_forward(x, 0.6, tw, bws, O.token_positions(n_txt, grids), cfg)
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.abs(y - x).max() > 1e-3  # the blocks did something


def test_table_rotation_matches_the_oracle_rope():
    """The oracle ops' RoPE-from-table equals the oracle's RoPE from positions."""
    dims, cfg, *_ = _case(128, n_blocks=1)
    pos = O.token_positions(3, [(0, 4, 5), (2, 3, 3)])
    ang = O.rope_angles(pos, cfg.rope_sections, cfg.rope_theta)
    table = np.stack([np.cos(ang), np.sin(ang)], axis=-1)
    x = np.random.default_rng(0).standard_normal((pos.shape[0], 2, cfg.head_dim))
    got = rotate_with_table(x, table, cfg.rope_sections)
    assert np.allclose(got, O.apply_rope(x, pos, cfg.rope_sections, cfg.rope_theta),
                       rtol=0, atol=1e-13)


def test_partition_rules():
    from image_generation_b200.ulysses import UlyssesRank

    ops = OracleOps(None, None, None)
    with pytest.raises(ValueError):
        UlyssesRank(ops, 0, 3, 288, 768, 8, 96, 2048)   # 3 ranks, 8 heads
    with pytest.raises(ValueError):
        UlyssesRank(ops, 0, 5, 288, 768, 10, 96, 2048)  # 288 tokens over 5 ranks
    r = UlyssesRank(ops, 2, 4, 288, 768, 8, 96, 2048)
    assert r.rows() == slice(144, 216) and r.cw == 192


# ---------------------------------------------------------------- fused form
# The fused exchanges (h3dit_sp_qkv_scatter / h3dit_sp_attention_scatter)
# write into other ranks' buffers. Here the ranks are gloo processes whose
# exchange buffers live in one shared-memory arena, the CPU stand-in for
# peer memory: a rank's "IPC handle" names the arena and a byte offset, and
# the oracle ops below store into the addresses they are given, with the
# layouts include/h3dit.h documents for the two calls.

class ArenaIpc:
    def __init__(self, arena):
        self.arena, self.opened = arena, 0

    def handle(self, t):
        return b"arena", t.data_ptr() - self.arena.data_ptr()

    def open(self, h):
        assert h == b"arena"
        self.opened += 1
        return self.arena.data_ptr()

    def close(self, base):
        assert base == self.arena.data_ptr()


class ArenaOracleOps(OracleOps):
    """OracleOps whose "exchange" buffers are carved from the shared arena
    (rank r's at its own offsets) and whose fused-exchange calls write to
    arena addresses."""

    def __init__(self, cfg, tw, bws, arena, rank, per_rank):
        super().__init__(cfg, tw, bws)
        self.arena, self.next = arena, rank * per_rank

    def empty(self, shape, kind):
        if kind != "exchange":
            return super().empty(shape, kind)
        size = int(np.prod(shape))
        v = self.arena[self.next:self.next + size].view(*shape)
        self.next += size
        return v

    def _at(self, ptr, shape):
        off = ptr - self.arena.data_ptr()
        assert off % 8 == 0 and off >= 0
        i = off // 8
        return self.arena[i:i + int(np.prod(shape))].view(*shape)

    def sp_qkv_scatter(self, xm, w_qkv, rope_rows, recv_ptrs, rank):
        n, I, P = xm.shape[0], self.cfg.inner, len(recv_ptrs)
        cw = I // P
        y = torch.empty(n, 3 * I, dtype=torch.float64)
        self.linear(EPI_QKV_ROPE, xm, w_qkv, y, rope_table=rope_rows)
        for g, ptr in enumerate(recv_ptrs):
            dst = self._at(ptr, (P * n, 3 * cw))
            for m in range(3):
                dst[rank * n:(rank + 1) * n, m * cw:(m + 1) * cw] = \
                    y[:, m * I + g * cw:m * I + (g + 1) * cw]

    def sp_attention_scatter(self, recv, o_ptrs, rank):
        n_all, P = recv.shape[0], len(o_ptrs)
        cw, n = self.cfg.inner // P, recv.shape[0] // len(o_ptrs)
        o_heads = torch.empty(n_all, cw, dtype=torch.float64)
        self.attention_heads(self.cfg.heads // P, recv[:, :cw], recv[:, cw:2 * cw],
                             recv[:, 2 * cw:], 3 * cw, o_heads, cw, n_all)
        for p, ptr in enumerate(o_ptrs):
            dst = self._at(ptr, (n, self.cfg.inner))
            dst[:, rank * cw:(rank + 1) * cw] = o_heads[p * n:(p + 1) * n]


def _fused_sizes(dims, n_total, world):
    cw = dims.heads * dims.head_dim // world
    return n_total * 3 * cw + (n_total // world) * dims.heads * dims.head_dim


def _fused_rank_main(rank, world, port, head_dim, arena, out):
    import torch.distributed as dist

    from image_generation_b200.ulysses import UlyssesStep

    torch.set_num_threads(2)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dims, cfg, tw, bws, n_txt, grids, x = _case(head_dim)
        n_total = x.shape[0]
        ops = ArenaOracleOps(cfg, tw, bws, arena, rank, _fused_sizes(dims, n_total, world))
        ipc = ArenaIpc(arena)
        step = UlyssesStep(ops, [dict(b) for b in bws], rank, world, n_total, dims.hidden,
                           dims.heads, dims.head_dim, dims.ffn, fused=True,
                           barrier=dist.barrier, ipc=ipc)
        # each peer's two exchange buffers sit in one allocation (the arena),
        # which is opened once per peer
        assert ipc.opened == world - 1
        assert step.r.recv_ptrs[rank] == step.r.recv.data_ptr()
        xl = torch.from_numpy(x[step.r.rows()].copy())
        step(0.6, xl, grids, n_txt)
        dist.barrier()
        step.close(ipc)
        rows = [torch.empty_like(xl) for _ in range(world)]
        dist.all_gather(rows, xl)
        if rank == 0:
            out["y"] = torch.cat(rows).numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,head_dim", [(2, 96), (4, 96), (2, 128)],
                         ids=["sp2", "sp4", "sp2_dh128"])
def test_fused_exchange_ranks_match_the_unsharded_step(world, head_dim):
    """The fused form: no all-to-all and no re-layout; each rank's QKV and
    attention write straight into the other ranks' buffers (here a shared
    arena), ordered by a barrier after each stage."""
    dims, cfg, tw, bws, n_txt, grids, x = _case(head_dim)
    arena = torch.full((world * _fused_sizes(dims, x.shape[0], world),), float("nan"),
                       dtype=torch.float64).share_memory_()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_fused_rank_main, args=(r, world, port, head_dim, arena, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        y = out["y"]
    ref = O.step_forward(x, 0.6, tw, bws, O.token_positions(n_txt, grids), cfg)
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.abs(y - x).max() > 1e-3


def test_fused_partition_rules():
    from image_generation_b200.ulysses import FusedUlyssesRank

    ops = OracleOps(None, None, None)
    with pytest.raises(ValueError):
        FusedUlyssesRank(ops, 0, 16, 288, 768, 16, 96, 2048)  # more ranks than addressable
    with pytest.raises(ValueError):
        FusedUlyssesRank(ops, 0, 3, 288, 768, 8, 96, 2048)    # 3 ranks, 8 heads
    r = FusedUlyssesRank(ops, 1, 4, 288, 768, 8, 96, 2048)
    assert tuple(r.recv.shape) == (288, 3 * 192) and tuple(r.o.shape) == (72, 768)
    with pytest.raises(ValueError):
        r.connect([0, 1, 2], [0, 1, 2, 3])
