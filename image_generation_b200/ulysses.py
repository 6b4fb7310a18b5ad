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

`ops` is the binding's Context, or any object with the same methods and an
`empty(shape, kind)` allocator (kind "act" for the token-major activations,
"f32" for fp32 vectors, "rope" for the RoPE table); the tests use an oracle-
backed one on the CPU to check the partition with real gloo ranks.
"""
from __future__ import annotations

from typing import Callable, Sequence

H3DIT_EPI_QKV_ROPE = 1
H3DIT_EPI_GELU = 2
H3DIT_EPI_GATED_RESIDUAL = 3


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


class UlyssesStep:
    """A sampling step under Ulysses SP on this rank: the timestep MLP, every
    block's AdaLN projection and the sequence's RoPE table are computed on
    every rank (they are small and need no exchange), then the blocks."""

    def __init__(self, ops, weights: Sequence[dict], rank: int, world: int, n_total: int,
                 hidden: int, heads: int, head_dim: int, ffn: int,
                 all_to_all: Callable | None = None, group=None):
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
            block(self.r, x, self.mod[l], w, rope_rows, self.all_to_all)
