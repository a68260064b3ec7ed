"""Sequence parallelism over attention heads (Ulysses) for the DiT.

"Wan（通义万相）..." 5.2 scales the DiT over many GPUs with a two-level context
parallelism: an inner level that splits the attention heads across the GPUs
of a node (Ulysses) and an outer level that splits the sequence and passes
key/value blocks around a ring.  This module is the inner level.

Each of N ranks holds a contiguous slice of n = L / N tokens of the residual
stream.  Everything in a block is row-local except the self-attention, which
needs every token.  So per block:

1. wd_block_qkv on the rank's token slice -> q|k|v [B, n, 3D] (RoPE uses the
   tokens' places in the whole grid);
2. all-to-all: rank r sends head group g (heads g*h/N .. (g+1)*h/N - 1, their
   q, k and v columns) of its tokens to rank g and receives its own head
   group for every token -> q|k|v [B, L, 3D/N];
3. wd_block_self_attention over the whole sequence for those h/N heads ->
   o [B, L, D/N];
4. all-to-all back: the attention output of token slice s goes to rank s ->
   o [B, n, D] with every head;
5. wd_block_post on the token slice (output projection, cross-attention,
   FFN).

The exchanges move 3 * B * n * D + B * n * D elements per rank per block; the
arithmetic is exactly that of the single-GPU block (same kernels on the same
rows), so the result is bit-identical to wd_block_forward.  The exchange is a
callable `exchange(recv, send)` with the semantics of
torch.distributed.all_to_all_single on dimension 0 (NCCL between GPUs); the
remote data lands in local memory before any kernel reads it.
"""
from __future__ import annotations

import torch


def token_slices(L: int, world: int):
    """(first token, count) of each rank's slice: equal contiguous slices."""
    if L % world:
        raise ValueError(f"{L} tokens do not split evenly over {world} ranks")
    n = L // world
    return [(r * n, n) for r in range(world)]


# ------------------------------------------------------------------ layout of the two exchanges
def heads_send(qkv: torch.Tensor, world: int) -> torch.Tensor:
    """q|k|v of this rank's tokens [B, n, 3D] -> [world, B, n, 3, D/world]:
    chunk g holds the q, k and v columns of head group g."""
    B, n, D3 = qkv.shape
    D = D3 // 3
    return qkv.view(B, n, 3, world, D // world).permute(3, 0, 1, 2, 4).contiguous()


def heads_recv(recv: torch.Tensor) -> torch.Tensor:
    """[world (source slice s), B, n, 3, Dg] -> q|k|v of one head group for the
    whole sequence [B, world * n, 3 * Dg] (tokens in slice order; columns q of
    the group's heads, then k, then v)."""
    world, B, n, _, Dg = recv.shape
    return recv.permute(1, 0, 2, 3, 4).reshape(B, world * n, 3 * Dg)


def tokens_send(o: torch.Tensor, world: int) -> torch.Tensor:
    """Attention output of one head group [B, L, Dg] -> [world, B, n, Dg]:
    chunk s holds token slice s."""
    B, L, Dg = o.shape
    return o.view(B, world, L // world, Dg).permute(1, 0, 2, 3).contiguous()


def tokens_recv(recv: torch.Tensor) -> torch.Tensor:
    """[world (source head group g), B, n, Dg] -> this slice's attention
    output with every head [B, n, world * Dg]."""
    world, B, n, Dg = recv.shape
    return recv.permute(1, 2, 0, 3).reshape(B, n, world * Dg)


class UlyssesBlock:
    """One rank's part of a block under head-sharded sequence parallelism.

    ops: the three pieces of a block for this rank's data,
      ops.qkv(blk, tok0, n, X_local) -> q|k|v [B, n, 3D]
      ops.attention(qkv_heads, heads) -> o [B, L, heads * dh]
      ops.post(blk, o_local, X_local)   (X_local updated in place)
    The stages are separate methods so that the same orchestration can be
    driven rank by rank (several ranks emulated in one process) or, through
    forward(), with a real all-to-all."""

    def __init__(self, ops, rank: int, world: int, L: int, heads: int):
        if heads % world:
            raise ValueError(f"{heads} heads do not split evenly over {world} ranks")
        self.ops, self.rank, self.world = ops, rank, world
        self.tok0, self.n = token_slices(L, world)[rank]
        self.heads_local = heads // world

    def stage_qkv(self, blk: int, X_local: torch.Tensor) -> torch.Tensor:
        return heads_send(self.ops.qkv(blk, self.tok0, self.n, X_local), self.world)

    def stage_attention(self, recv_qkv: torch.Tensor) -> torch.Tensor:
        return tokens_send(self.ops.attention(heads_recv(recv_qkv), self.heads_local), self.world)

    def stage_post(self, blk: int, recv_o: torch.Tensor, X_local: torch.Tensor):
        self.ops.post(blk, tokens_recv(recv_o), X_local)

    def forward(self, blk: int, X_local: torch.Tensor, exchange) -> torch.Tensor:
        send = self.stage_qkv(blk, X_local)
        recv = torch.empty_like(send)
        exchange(recv, send)
        send = self.stage_attention(recv)
        recv = torch.empty_like(send)
        exchange(recv, send)
        self.stage_post(blk, recv, X_local)
        return X_local


def block_in_one_process(blocks, X_locals, blk: int):
    """Run block `blk` for all ranks' UlyssesBlocks in this process, one rank
    after the other, the all-to-all done by copying: rank r receives, from
    every rank s, chunk r of s's send buffer.  For checking the orchestration
    without several processes (no rank ever waits for another)."""
    def a2a(sends):
        return [torch.stack([sends[s][r] for s in range(len(sends))]) for r in range(len(sends))]
    recv = a2a([b.stage_qkv(blk, X) for b, X in zip(blocks, X_locals)])
    recv = a2a([b.stage_attention(rv) for b, rv in zip(blocks, recv)])
    for b, rv, X in zip(blocks, recv, X_locals):
        b.stage_post(blk, rv, X)


def nccl_exchange(group=None):
    """exchange(recv, send) = all_to_all_single over `group` (dimension 0)."""
    import torch.distributed as dist

    def ex(recv, send):
        dist.all_to_all_single(recv, send, group=group)
    return ex


class LibwdOps:
    """The three pieces on one GPU through libwd, for a batch-B model whose
    weights, context K/V and workspace live in `net` (a model.DiT)."""

    def __init__(self, net):
        from . import wd
        self.wd, self.net = wd, net

    def qkv(self, blk, tok0, n, X_local):
        net = self.net
        out = torch.empty((net.batch, n, 3 * net.dims.D), dtype=net.tdtype, device=X_local.device)
        self.wd.wd_block_qkv(net.cd, net.block_w[blk], net.e0, net.batch, tok0, n, X_local, out, net.ws)
        return out

    def attention(self, qkv_heads, heads):
        net = self.net
        B, L, _ = qkv_heads.shape
        o = torch.empty((B, L, heads * net.dims.dh), dtype=net.tdtype, device=qkv_heads.device)
        self.wd.wd_block_self_attention(net.cd, B, heads, qkv_heads, o)
        return o

    def post(self, blk, o_local, X_local):
        net = self.net
        self.wd.wd_block_post(net.cd, net.block_w[blk], net.e0, net.kv[blk], net.batch, X_local.shape[1],
                              o_local.contiguous(), X_local, net.ws)


class SeqParallelDiT:
    """A whole DiT forward with the blocks under Ulysses sequence parallelism
    on `world` GPUs (one process each).  Every rank holds the full model
    (weights, context K/V) and the full-size buffers of `net`; the time MLP
    and the patch embedding run on every rank (they are tiny), each rank keeps
    its token slice of the residual stream through the blocks, and an
    all-gather of the slices before the head gives every rank the velocity."""

    def __init__(self, net, rank: int, world: int, group=None, exchange=None):
        import torch.distributed as dist
        self.net, self.rank, self.world, self.group = net, rank, world, group
        d = net.dims
        self.block = UlyssesBlock(LibwdOps(net), rank, world, d.L, d.heads)
        self.exchange = exchange or nccl_exchange(group)
        self._dist = dist
        B, n = net.batch, self.block.n
        self.X_local = torch.empty((B, n, d.D), dtype=torch.float32, device=net.X.device)
        self._gather = torch.empty((world, B, n, d.D), dtype=torch.float32, device=net.X.device)

    def forward(self, x_t, y, tau: float):
        from . import wd
        net, blk = self.net, self.block
        wd.wd_time_mod(net.cd, net.time_w, tau, net.e, net.e0)
        wd.wd_patch_embed(net.cd, x_t, y, net.w["pe.w"], net.w["pe.b"], net.batch, net.X, net.ws)
        self.X_local.copy_(net.X[:, blk.tok0:blk.tok0 + blk.n])
        for i in range(net.dims.blocks):
            blk.forward(i, self.X_local, self.exchange)
        self._dist.all_gather_into_tensor(self._gather, self.X_local.unsqueeze(0).contiguous(), group=self.group)
        net.X.copy_(self._gather.permute(1, 0, 2, 3).reshape(net.X.shape))
        wd.wd_unpatchify(net.cd, net.head_w, net.e, net.batch, net.X, net.v, net.ws)
        return net.v

    def cfg_euler_step(self, xb: torch.Tensor, y, tau: float, dt: float, cfg_scale: float) -> torch.Tensor:
        """One CFG Euler step on xb [2, 16, T, H, W] (row 0 the text row, row 1
        the zeroed-text row; the model's context was prepared so): every rank
        ends with the same updated latent in both rows."""
        from . import wd
        v = self.forward(xb, y, tau)
        wd.wd_euler_cfg_step(xb[0], v[0], v[1], cfg_scale, dt)
        xb[1].copy_(xb[0])
        return xb
