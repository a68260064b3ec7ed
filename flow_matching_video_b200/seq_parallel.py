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
    """A whole DiT forward with the blocks under context parallelism on
    `world` GPUs (one process each): Ulysses over all of them (ring = 1), or
    the two-level scheme with `ring` groups of world / ring ranks.  Every rank
    holds the full model (weights, context K/V) and the full-size buffers of
    `net`; the time MLP and the patch embedding run on every rank (they are
    tiny), each rank keeps its token slice of the residual stream through the
    blocks, and an all-gather of the slices before the head gives every rank
    the velocity.  Every rank must construct it (it creates the process groups
    of the two levels in the same order on all ranks)."""

    def __init__(self, net, rank: int, world: int, group=None, exchange=None, ring: int = 1):
        import torch.distributed as dist
        self.net, self.rank, self.world, self.group = net, rank, world, group
        d = net.dims
        self._dist = dist
        if world % ring:
            raise ValueError(f"{world} ranks do not form {ring} ring groups")
        self.ring = ring
        if ring == 1:
            self.block = UlyssesBlock(LibwdOps(net), rank, world, d.L, d.heads)
            self.exchange = exchange or nccl_exchange(group)
        else:
            U = world // ring
            ul, _ = cp2d_groups(U, ring)
            self.block = CP2DBlock(LibwdRingOps(net), rank, U, ring, d.L, d.heads)
            self.exchange = exchange or nccl_exchange(ul[self.block.g])
            self.ring_pass = ring_pass_fn(rank, U, ring)
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
            if self.ring == 1:
                blk.forward(i, self.X_local, self.exchange)
            else:
                blk.forward(i, self.X_local, self.exchange, self.ring_pass)
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


# ------------------------------------------------------------------ 2D context parallelism: Ulysses x ring
class CP2DBlock:
    """One rank's part of a block under the two-level context parallelism of
    "Wan（通义万相）..." 5.2: U ranks per Ulysses group (heads split inside the
    group) times R groups on a ring (the sequence split across groups).

    Rank r = g * U + u holds token slice r of L / (U R) tokens.  Group g's U
    slices form chunk g (L / R tokens).  Per block:
      1. q|k|v of the rank's slice (RoPE at the tokens' places in the grid);
      2. all-to-all inside the group: head group u of chunk g -> [B, L/R, 3D/U];
      3. the ring: the R ranks with the same u pass their chunks' keys and
         values around; at step s a rank attends its queries (chunk g) to the
         keys of chunk g - s and merges the result by log-sum-exp;
      4. all-to-all back inside the group: the slice's output with every head;
      5. the rest of the block on the slice.
    With R = 1 it is the Ulysses block; with U = 1 a pure ring.

    ops: qkv / post as for UlyssesBlock, plus
      ops.attention_lse(q, k, v, heads) -> (o [B, m, heads*dh], lse [B, heads, m])
      ops.merge(o_run, lse_run, o_part, lse_part, first, out)   (in place)
      ops.merge_state(q, heads) -> (o_run fp32, lse_run fp32) buffers"""

    def __init__(self, ops, rank: int, U: int, R: int, L: int, heads: int):
        if heads % U:
            raise ValueError(f"{heads} heads do not split evenly over {U} ranks")
        self.ops, self.U, self.R = ops, U, R
        self.g, self.u = divmod(rank, U)
        self.tok0, self.n = token_slices(L, U * R)[rank]
        self.heads_local = heads // U

    # the Ulysses exchanges are those of UlyssesBlock, inside the group
    def stage_qkv(self, blk: int, X_local: torch.Tensor) -> torch.Tensor:
        return heads_send(self.ops.qkv(blk, self.tok0, self.n, X_local), self.U)

    def ring_begin(self, recv_qkv: torch.Tensor):
        """-> (q [B, m, Dg], kv [2, B, m, Dg]) of this group's chunk for this head group."""
        qkv = heads_recv(recv_qkv)
        Dg = qkv.shape[2] // 3
        q = qkv[:, :, :Dg].contiguous()
        kv = torch.stack([qkv[:, :, Dg:2 * Dg], qkv[:, :, 2 * Dg:]]).contiguous()
        return q, kv

    def ring_step(self, q: torch.Tensor, kv: torch.Tensor, state, step: int):
        """Merge the attention of q to the keys/values kv into state (o_run,
        lse_run, out); the last step also writes the merged output, in the
        storage type, to out."""
        o, lse = self.ops.attention_lse(q, kv[0], kv[1], self.heads_local)
        if state is None:
            state = self.ops.merge_state(q, self.heads_local) + (torch.empty_like(q),)
        self.ops.merge(state[0], state[1], o, lse, step == 0, state[2] if step == self.R - 1 else None)
        return state

    def ring_end(self, state) -> torch.Tensor:
        """The merged output -> the send buffer of the return all-to-all."""
        return tokens_send(state[2], self.U)

    def stage_post(self, blk: int, recv_o: torch.Tensor, X_local: torch.Tensor):
        self.ops.post(blk, tokens_recv(recv_o), X_local)

    def forward(self, blk: int, X_local: torch.Tensor, a2a, ring_pass) -> torch.Tensor:
        """a2a(recv, send): all_to_all_single inside the Ulysses group;
        ring_pass(kv) -> the kv of the previous rank on the ring (this rank's
        kv goes to the next)."""
        send = self.stage_qkv(blk, X_local)
        recv = torch.empty_like(send)
        a2a(recv, send)
        q, kv = self.ring_begin(recv)
        state = None
        for s in range(self.R):
            state = self.ring_step(q, kv, state, s)
            if s + 1 < self.R:
                kv = ring_pass(kv)
        send = self.ring_end(state)
        recv = torch.empty_like(send)
        a2a(recv, send)
        self.stage_post(blk, recv, X_local)
        return X_local


def cp2d_block_in_one_process(blocks, X_locals, blk: int):
    """All U x R ranks of CP2DBlock in this process, one after the other: the
    all-to-alls by copying inside each group, the ring by handing each group's
    keys and values to the next group (for checking without several processes;
    no rank waits for another)."""
    U, R = blocks[0].U, blocks[0].R

    def a2a_groups(sends):
        out = [None] * (U * R)
        for g in range(R):
            grp = list(range(g * U, (g + 1) * U))
            for j, r in enumerate(grp):
                out[r] = torch.stack([sends[s][j] for s in grp])
        return out
    recv = a2a_groups([b.stage_qkv(blk, X) for b, X in zip(blocks, X_locals)])
    qs, kvs = zip(*[b.ring_begin(rv) for b, rv in zip(blocks, recv)])
    kvs = list(kvs)
    states = [None] * (U * R)
    for s in range(R):
        states = [b.ring_step(q, kv, st, s) for b, q, kv, st in zip(blocks, qs, kvs, states)]
        # rank g*U + u receives the kv of rank ((g - 1) mod R)*U + u
        kvs = [kvs[((r // U - 1) % R) * U + r % U] for r in range(U * R)]
    recv = a2a_groups([b.ring_end(st) for b, st in zip(blocks, states)])
    for b, rv, X in zip(blocks, recv, X_locals):
        b.stage_post(blk, rv, X)


def cp2d_groups(U: int, R: int):
    """The process groups of the two levels (every rank must call this, in the
    same order): the Ulysses groups {g U .. g U + U - 1} and the ring groups
    {u, U + u, ...}.  Returns (ulysses_groups, ring_groups)."""
    import torch.distributed as dist
    ul = [dist.new_group(list(range(g * U, (g + 1) * U))) for g in range(R)]
    rg = [dist.new_group(list(range(u, U * R, U))) for u in range(U)]
    return ul, rg


def ring_pass_fn(rank: int, U: int, R: int):
    """ring_pass(kv): send kv to the next rank on this rank's ring, receive the
    previous rank's (point-to-point, both posted before either is waited on)."""
    import torch.distributed as dist
    g, u = divmod(rank, U)
    nxt, prv = ((g + 1) % R) * U + u, ((g - 1) % R) * U + u

    def ring_pass(kv):
        recv = torch.empty_like(kv)
        reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, kv, nxt), dist.P2POp(dist.irecv, recv, prv)])
        for q in reqs:
            q.wait()
        return recv
    return ring_pass


class LibwdRingOps(LibwdOps):
    """LibwdOps plus the ring's attention with log-sum-exp and its merge."""

    def attention_lse(self, q, k, v, heads):
        net, wd = self.net, self.wd
        B, m, Dh = q.shape
        o = torch.empty_like(q)
        lse = torch.empty((B, heads, m), dtype=torch.float32, device=q.device)
        dt = wd.WD_BF16 if q.dtype == torch.bfloat16 else wd.WD_F32
        wd.wd_attention_lse(dt, B, m, heads, Dh // heads, q, k, v, k.shape[1], 0, o, lse)
        return o, lse

    def merge_state(self, q, heads):
        B, m, Dh = q.shape
        return (torch.empty((B, m, Dh), dtype=torch.float32, device=q.device),
                torch.empty((B, heads, m), dtype=torch.float32, device=q.device))

    def merge(self, o_run, lse_run, o_part, lse_part, first, out=None):
        wd = self.wd
        B, m, Dh = o_part.shape
        heads = lse_part.shape[1]
        dt = wd.WD_BF16 if o_part.dtype == torch.bfloat16 else wd.WD_F32
        wd.wd_attention_merge(dt, B, m, heads, Dh // heads, o_run, lse_run, o_part, lse_part, first, out)

