"""Ulysses sequence parallelism of the DiT step over P ranks.

"H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin", "Faster DiT" (Ulysses
SP4 distributes the sequence work over four GPUs) and the vLLM-Omni recipe's
"Deployment profiles" (Ulysses SP 2 and SP 4 rows). The partition:

  * rank r holds tokens [r n, (r + 1) n) of the packed sequence [text;
    images], n = N / P, as its slice of the fp32 residual stream, and runs the
    row-wise steps on them with all heads: RMSNorm + modulate, QKV + RoPE (on
    its rows of the sequence's RoPE table), out-projection, FFN;
  * around the attention, all-to-all #1 trades the rows' Q|K|V of every head
    for all N tokens' Q|K|V of heads r H/P .. (r + 1) H/P - 1, the attention
    runs on that head group, and all-to-all #2 sends each rank's token rows
    of the attention output back.

Every step of the block runs in libh3dit's kernels through the binding
(h3dit_sp_pack_qkv / h3dit_sp_unpack_o are the re-layouts on either side of
the exchanges, h3dit_attention_heads the attention on a head group); this
module holds the buffers, slices the sequence and calls the collective it is
given - torch.distributed.all_to_all_single (NCCL) between GPUs. Nothing here
computes any of the method's arithmetic.

The fused form (FusedUlyssesRank, fused_block) does the same exchanges with
no collective and no re-layout kernel: the QKV GEMM's epilogue stores each
head group's Q|K|V straight into the receive buffer of the rank that attends
over it, and the attention's epilogue stores each output row straight into
the out-projection input of the rank that holds the token
(h3dit_sp_qkv_scatter / h3dit_sp_attention_scatter). Between GPUs the
buffers are peer memory mapped with CUDA IPC (connect_peers), and a barrier
after each of the two stages orders the writes against the reads.

`ops` is the binding's Context, or any object with the same methods and an
`empty(shape, kind)` allocator (kind "act" for the token-major activations,
"exchange" for activations other ranks write into, "f32" for fp32 vectors,
"rope" for the RoPE table); the tests use an oracle-
backed one on the CPU to check the partition with real gloo ranks.
"""
from __future__ import annotations

from typing import Callable, Sequence

H3DIT_EPI_QKV_ROPE = 1
H3DIT_EPI_GELU = 2
H3DIT_EPI_GATED_RESIDUAL = 3
H3DIT_LINEAR_OUT, H3DIT_LINEAR_FFN1, H3DIT_LINEAR_FFN2 = 1, 2, 3


class UlyssesRank:
    """One rank's buffers and its three stages of a block."""

    def __init__(self, ops, rank: int, world: int, n_total: int, hidden: int, heads: int,
                 head_dim: int, ffn: int):
        if n_total % world:
            raise ValueError(f"{world} ranks do not divide {n_total} tokens")
        if heads % world:
            raise ValueError(f"{world} ranks do not divide {heads} heads")
        self.ops, self.rank, self.world = ops, rank, world
        self.n_total, self.n = n_total, n_total // world
        self.D, self.H, self.dh, self.F = hidden, heads, head_dim, ffn
        self.I = heads * head_dim
        self.cw = self.I // world  # columns of one head group per matrix
        e = ops.empty
        n, P = self.n, world
        self.xm = e((n, hidden), "act")
        self.qkv = e((n, 3 * self.I), "act")
        self.send1 = e((P, n, 3 * self.cw), "act")
        self.recv1 = e((P, n, 3 * self.cw), "act")
        self.o_heads = e((n_total, self.cw), "act")
        self.recv2 = e((P, n, self.cw), "act")
        self.o = e((n, self.I), "act")
        self.u = e((n, ffn), "act")

    def rows(self):
        """This rank's token rows of the packed sequence."""
        return slice(self.rank * self.n, (self.rank + 1) * self.n)

    def qkv_and_pack(self, x, mod, w, rope_rows):
        """RMSNorm + modulate, QKV + RoPE on this rank's rows, then the
        head-group blocks for all-to-all #1. Returns (send, recv)."""
        ops = self.ops
        ops.rmsnorm_modulate(x, mod[0], mod[1], self.xm)
        ops.linear(H3DIT_EPI_QKV_ROPE, self.xm, w["w_qkv"], self.qkv, rope_table=rope_rows)
        ops.sp_pack_qkv(self.qkv, self.world, self.send1)
        return self.send1, self.recv1

    def attention(self):
        """Attention of this rank's head group over all tokens; the output
        rows are the blocks of all-to-all #2. Returns (send, recv)."""
        cw, n_all = self.cw, self.n_total
        q = self.recv1.view(n_all, 3 * cw)
        self.ops.attention_heads(self.H // self.world, q[:, :cw], q[:, cw:2 * cw], q[:, 2 * cw:],
                                 3 * cw, self.o_heads, cw, n_all)
        return self.o_heads, self.recv2

    def finish(self, x, mod, w):
        """Back to row-major heads, out-projection with the gated residual,
        then the FFN branch, on this rank's rows (x updated in place)."""
        ops = self.ops
        ops.sp_unpack_o(self.recv2, self.world, self.o)
        ops.linear(H3DIT_EPI_GATED_RESIDUAL, self.o, w["w_o"], x, gate=mod[2])
        ops.rmsnorm_modulate(x, mod[3], mod[4], self.xm)
        ops.linear(H3DIT_EPI_GELU, self.xm, w["w_ff1"], self.u)
        ops.linear(H3DIT_EPI_GATED_RESIDUAL, self.u, w["w_ff2"], x, gate=mod[5])


def block(rank: UlyssesRank, x, mod, w, rope_rows, all_to_all: Callable) -> None:
    """One block on this rank's rows x (fp32 [n, D], in place);
    all_to_all(recv, send) exchanges equal blocks along the first axis."""
    send, recv = rank.qkv_and_pack(x, mod, w, rope_rows)
    all_to_all(recv, send)
    send, recv = rank.attention()
    all_to_all(recv, send)
    rank.finish(x, mod, w)


class FusedUlyssesRank:
    """One rank's buffers for the fused exchanges: `recv` [N, 3I/P] receives
    the Q|K|V of this rank's heads from every rank's QKV GEMM, and `o`
    [N/P, I] receives this rank's token rows of the attention output from
    every rank's attention. `connect` takes every rank's `recv` and `o`
    device addresses in rank order (its own included).

    With mx=True the block runs the MXFP8 linears of an MXFP8 context (the
    context's quantized weights, so the stages take the block's index): the
    rows are quantized by the MXFP8 RMSNorm, `o` holds E4M3 codes and
    `o_sf` their scales, which every rank's attention writes too; `recv`
    stays bf16."""

    def __init__(self, ops, rank: int, world: int, n_total: int, hidden: int, heads: int,
                 head_dim: int, ffn: int, max_ranks: int = 8, mx: bool = False):
        if not 1 <= world <= max_ranks:
            raise ValueError(f"the fused exchange addresses 1 .. {max_ranks} ranks, not {world}")
        if n_total % world:
            raise ValueError(f"{world} ranks do not divide {n_total} tokens")
        if heads % world:
            raise ValueError(f"{world} ranks do not divide {heads} heads")
        self.ops, self.rank, self.world = ops, rank, world
        self.n_total, self.n = n_total, n_total // world
        self.D, self.H, self.dh, self.F = hidden, heads, head_dim, ffn
        self.I = heads * head_dim
        self.cw = self.I // world
        self.mx = mx
        e = ops.empty
        self.recv = e((n_total, 3 * self.cw), "exchange")  # written by every rank
        if mx:
            sf = ops.mx_scale_bytes
            self.xm = e((self.n, hidden), "fp8")
            self.xm_sf = e((sf(self.n, hidden),), "sf")
            self.o = e((self.n, self.I), "exchange_fp8")          # written by every rank
            self.o_sf = e((sf(self.n, self.I),), "exchange_sf")   # written by every rank
            self.u = e((self.n, ffn), "fp8")
            self.u_sf = e((sf(self.n, ffn),), "sf")
        else:
            self.xm = e((self.n, hidden), "act")
            self.o = e((self.n, self.I), "exchange")            # written by every rank
            self.u = e((self.n, ffn), "act")
        self.recv_ptrs: list | None = None
        self.o_ptrs: list | None = None
        self.o_sf_ptrs: list | None = None

    def exchanged(self) -> list:
        """The buffers other ranks write into, in the order connect takes
        their addresses."""
        return [self.recv, self.o] + ([self.o_sf] if self.mx else [])

    def rows(self):
        return slice(self.rank * self.n, (self.rank + 1) * self.n)

    def connect(self, recv_ptrs: Sequence[int], o_ptrs: Sequence[int],
                o_sf_ptrs: Sequence[int] | None = None) -> None:
        if len(recv_ptrs) != self.world or len(o_ptrs) != self.world:
            raise ValueError("one receive and one output address per rank")
        if self.mx and (o_sf_ptrs is None or len(o_sf_ptrs) != self.world):
            raise ValueError("one scale-array address per rank")
        self.recv_ptrs, self.o_ptrs = list(recv_ptrs), list(o_ptrs)
        self.o_sf_ptrs = None if o_sf_ptrs is None else list(o_sf_ptrs)

    def qkv_scatter(self, x, mod, w, rope_rows, block: int = 0) -> None:
        """RMSNorm + modulate, then QKV + RoPE with the first exchange fused
        in: every rank's `recv` gets this rank's rows of its head group."""
        if self.mx:
            self.ops.rmsnorm_modulate_mx(x, mod[0], mod[1], self.xm, self.xm_sf)
            self.ops.sp_qkv_scatter_mx(self.xm, self.xm_sf, block, rope_rows, self.recv_ptrs,
                                       self.rank)
            return
        self.ops.rmsnorm_modulate(x, mod[0], mod[1], self.xm)
        self.ops.sp_qkv_scatter(self.xm, w["w_qkv"], rope_rows, self.recv_ptrs, self.rank)

    def attention_scatter(self) -> None:
        """Attention of this rank's heads over all tokens, with the second
        exchange fused in: every rank's `o` gets its rows for these heads."""
        if self.mx:
            self.ops.sp_attention_scatter_mx(self.recv, self.o_ptrs, self.o_sf_ptrs, self.rank)
            return
        self.ops.sp_attention_scatter(self.recv, self.o_ptrs, self.rank)

    def finish(self, x, mod, w, block: int = 0) -> None:
        ops = self.ops
        if self.mx:
            ops.block_linear_mx(block, H3DIT_LINEAR_OUT, self.o, self.o_sf, x, gate=mod[2])
            ops.rmsnorm_modulate_mx(x, mod[3], mod[4], self.xm, self.xm_sf)
            ops.block_linear_mx(block, H3DIT_LINEAR_FFN1, self.xm, self.xm_sf, self.u, self.u_sf)
            ops.block_linear_mx(block, H3DIT_LINEAR_FFN2, self.u, self.u_sf, x, gate=mod[5])
            return
        ops.linear(H3DIT_EPI_GATED_RESIDUAL, self.o, w["w_o"], x, gate=mod[2])
        ops.rmsnorm_modulate(x, mod[3], mod[4], self.xm)
        ops.linear(H3DIT_EPI_GELU, self.xm, w["w_ff1"], self.u)
        ops.linear(H3DIT_EPI_GATED_RESIDUAL, self.u, w["w_ff2"], x, gate=mod[5])


def fused_block(rank: FusedUlyssesRank, x, mod, w, rope_rows, barrier: Callable,
                block: int = 0) -> None:
    """One block with the fused exchanges (`block`: its index, which the
    MXFP8 form uses to find the context's quantized weights). barrier() must
    return only when every rank's work so far has completed on its GPU: after
    the first stage the attention reads what all ranks wrote, and after the
    second the out-projection does; the next block's first stage then
    overwrites `recv`, which every rank has finished reading by the second
    barrier."""
    rank.qkv_scatter(x, mod, w, rope_rows, block)
    barrier()
    rank.attention_scatter()
    barrier()
    rank.finish(x, mod, w, block)


def connect_peers(rank: FusedUlyssesRank, ipc=None, group=None) -> list:
    """Maps every other rank's `recv` and `o` into this process and connects
    the rank. Each buffer is named by (handle, byte offset, the allocation's
    base address in its owner); the names are exchanged with
    all_gather_object, and an allocation is opened once even when both
    buffers sit in it. `ipc` supplies handle(t) -> (bytes, offset),
    open(handle) -> base address and close(base) (the binding's CUDA IPC by
    default). Returns the opened base addresses, for close_peers."""
    import torch.distributed as dist

    if ipc is None:
        from . import h3dit as H

        ipc = _BindingIpc(H)

    def named(t):
        h, off = ipc.handle(t)
        return h, off, t.data_ptr() - off  # the allocation's base in the owner

    bufs = rank.exchanged()
    mine = [named(t) for t in bufs]
    everyone = [None] * rank.world
    dist.all_gather_object(everyone, mine, group=group)
    bases: dict = {}
    cols: list = [[] for _ in bufs]  # per buffer, every rank's address
    for r, names in enumerate(everyone):
        for i, (h, off, owner_base) in enumerate(names):
            if r == rank.rank:
                cols[i].append(bufs[i].data_ptr())
                continue
            key = (r, owner_base)  # one opening per allocation of each rank
            if key not in bases:
                bases[key] = ipc.open(h)
            cols[i].append(bases[key] + off)
    rank.connect(*cols)
    return list(bases.values())


def close_peers(bases: Sequence[int], ipc=None) -> None:
    if ipc is None:
        from . import h3dit as H

        ipc = _BindingIpc(H)
    for b in bases:
        ipc.close(b)


class _BindingIpc:
    def __init__(self, H):
        self.H = H

    def handle(self, t):
        return self.H.ipc_handle(t)

    def open(self, h):
        return self.H.ipc_open(h, 0)

    def close(self, base):
        self.H.ipc_close(base, 0)


def host_barrier(group=None) -> Callable:
    """The barrier fused_block needs between GPUs: this rank's stream
    drained, then a barrier across the ranks."""
    import torch
    import torch.distributed as dist

    def barrier():
        torch.cuda.current_stream().synchronize()
        dist.barrier(group=group)

    return barrier


class UlyssesStep:
    """A sampling step under Ulysses SP on this rank: the timestep MLP, every
    block's AdaLN projection and the sequence's RoPE table are computed on
    every rank (they are small and need no exchange), then the blocks."""

    def __init__(self, ops, weights: Sequence[dict], rank: int, world: int, n_total: int,
                 hidden: int, heads: int, head_dim: int, ffn: int,
                 all_to_all: Callable | None = None, group=None, fused: bool = False,
                 barrier: Callable | None = None, ipc=None, mx: bool = False):
        self.fused = fused
        self.peer_bases: list = []
        if mx and not fused:
            raise ValueError("the MXFP8 block runs with the fused exchanges")
        if fused:
            # collective: every rank constructs its step at the same point
            self.r = FusedUlyssesRank(ops, rank, world, n_total, hidden, heads, head_dim, ffn,
                                      mx=mx)
            self.peer_bases = connect_peers(self.r, ipc=ipc, group=group)
            self.barrier = barrier if barrier is not None else host_barrier(group)
        else:
            self.r = UlyssesRank(ops, rank, world, n_total, hidden, heads, head_dim, ffn)
        self.ops, self.weights = ops, list(weights)
        self.c = ops.empty((hidden,), "f32")
        self.mod = ops.empty((len(self.weights), 6, hidden), "f32")
        self.rope = ops.empty((n_total, head_dim // 2, 2), "rope")
        if all_to_all is None:
            import torch.distributed as dist

            all_to_all = lambda recv, send: dist.all_to_all_single(recv, send, group=group)
        self.all_to_all = all_to_all

    def __call__(self, t: float, x, grids, n_txt: int) -> None:
        """x: this rank's rows of the fp32 residual [N / P, D], in place."""
        ops = self.ops
        ops.time_embed(t, self.c)
        ops.adaln_project(self.c, 0, len(self.weights), self.mod)
        ops.rope_table(grids, n_txt, self.rope)
        rope_rows = self.rope[self.r.rows()]
        for l, w in enumerate(self.weights):
            if self.fused:
                fused_block(self.r, x, self.mod[l], w, rope_rows, self.barrier, block=l)
            else:
                block(self.r, x, self.mod[l], w, rope_rows, self.all_to_all)

    def close(self, ipc=None) -> None:
        """Unmaps the peers' buffers (fused form): call on every rank after
        the last step, once every rank has stopped writing."""
        close_peers(self.peer_bases, ipc)
        self.peer_bases = []
