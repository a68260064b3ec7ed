"""Head-sharded sequence parallelism (Ulysses, "Wan（通义万相）..." 5.2) on the CPU.

The orchestration of flow_matching_video_b200.seq_parallel (token slices,
the two all-to-all exchanges and their layouts) is driven with the oracle's
pieces of a block as the per-rank compute: block_qkv on a token slice, the
attention over a head group, block_after_attention on the slice.  The
gathered result must equal the oracle's block_forward on the whole sequence.
Ranks are emulated in one process and run as 2 and 4 gloo processes with a
real all_to_all_single.  No GPU needed.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import wan_oracle as O
from flow_matching_video_b200 import seq_parallel as SP
from flow_matching_video_b200 import synth


def tiny_case(seed=5):
    """A tiny fp64 block with 4 heads of 16 and a 2 x 2 x 3 token grid (L = 12,
    divisible by 2 and 4)."""
    d = synth.Dims(D=64, heads=4, ffn=48, blocks=1, T=2, H=4, W=6, n_txt=5, c_txt=12, n_img=4, c_img=10,
                   dtype="f32")
    wl = synth.Workload("sp", d, batch=2, seed=seed)
    w = {k: v.astype(np.float64) * (10 if k.endswith(".w") else 1) for k, v in synth.model_weights(wl).items()}
    rng = np.random.default_rng(seed)
    txt = rng.standard_normal((2, d.n_txt, d.c_txt))
    clip = rng.standard_normal((d.n_img, d.c_img))
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv = O.cross_kv(w, 0, ctx_t, ctx_i)
    X = rng.standard_normal((2, d.L, d.D))
    e0 = rng.standard_normal((6, d.D)) * 0.5
    return d, w, kv, X, e0


class OracleOps:
    """The three pieces of a block, computed by the oracle on torch float64 tensors."""

    def __init__(self, d, w, kv, e0):
        self.d, self.w, self.kv, self.e0 = d, w, kv, e0

    def qkv(self, blk, tok0, n, X_local):
        out = []
        for b in range(X_local.shape[0]):
            r = O.block_qkv(X_local[b].numpy(), self.e0, self.w, blk, self.d, np.arange(tok0, tok0 + n))
            out.append(np.concatenate([r[k].reshape(n, -1) for k in ("q", "k", "v")], axis=1))
        return torch.from_numpy(np.stack(out))

    def attention(self, qkv_heads, heads):
        B, L, D3 = qkv_heads.shape
        dh = D3 // (3 * heads)
        a = qkv_heads.numpy().reshape(B, L, 3, heads, dh)
        return torch.from_numpy(np.stack([O.attention(a[b, :, 0], a[b, :, 1], a[b, :, 2]).reshape(L, heads * dh)
                                          for b in range(B)]))

    def post(self, blk, o_local, X_local):
        X_local.copy_(torch.from_numpy(O.block_after_attention(X_local.numpy(), o_local.numpy(), self.e0, self.w,
                                                               blk, self.kv, self.d)))


@pytest.mark.parametrize("world", [1, 2, 4])
def test_ulysses_in_one_process_equals_the_whole_block(world):
    d, w, kv, X, e0 = tiny_case()
    want = O.block_forward(X, e0, w, 0, kv, d)
    ops = OracleOps(d, w, kv, e0)
    blocks = [SP.UlyssesBlock(ops, r, world, d.L, d.heads) for r in range(world)]
    X_locals = [torch.from_numpy(X[:, b.tok0:b.tok0 + b.n].copy()) for b in blocks]
    SP.block_in_one_process(blocks, X_locals, 0)
    got = torch.cat(X_locals, dim=1).numpy()
    np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)
    assert np.abs(got - X).max() > 1.0          # the block did move X


def test_ulysses_layouts_pick_the_right_heads_and_tokens():
    # labelled entries: the value encodes (batch, token, q/k/v, column)
    world, B, n, D = 2, 2, 3, 8
    qkv = torch.arange(B * n * 3 * D, dtype=torch.float64).view(B, n, 3 * D)
    send = SP.heads_send(qkv, world)                      # [world, B, n, 3, D/world]
    for g in range(world):
        for j in range(3):
            torch.testing.assert_close(send[g, :, :, j], qkv[:, :, j * D + g * D // world:j * D + (g + 1) * D // world])
    # two slices' sends -> one head group's whole sequence
    recv = torch.stack([send, send + 1000])[:, 0]          # from slices 0 and 1, head group 0
    full = SP.heads_recv(recv)
    assert full.shape == (B, world * n, 3 * D // world)
    torch.testing.assert_close(full[:, n:, :D // world], qkv[:, :, :D // world] + 1000)
    o = torch.arange(B * world * n * 4, dtype=torch.float64).view(B, world * n, 4)
    back = SP.tokens_recv(torch.stack([SP.tokens_send(o, world)[1], SP.tokens_send(o + 7, world)[1]]))
    torch.testing.assert_close(back, torch.cat([o[:, n:], o[:, n:] + 7], dim=2))


def test_ulysses_refuses_uneven_splits():
    with pytest.raises(ValueError):
        SP.token_slices(12, 5)
    with pytest.raises(ValueError):
        SP.UlyssesBlock(None, 0, 3, 12, 4)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        d, w, kv, X, e0 = tiny_case()
        blk = SP.UlyssesBlock(OracleOps(d, w, kv, e0), rank, world, d.L, d.heads)
        X_local = torch.from_numpy(X[:, blk.tok0:blk.tok0 + blk.n].copy())
        blk.forward(0, X_local, SP.nccl_exchange())
        out[rank] = X_local.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_gloo_ranks_equal_the_whole_block(world):
    d, w, kv, X, e0 = tiny_case()
    want = O.block_forward(X, e0, w, 0, kv, d)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        got = np.concatenate([out[r] for r in range(world)], axis=1)
    np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)


# ------------------------------------------------------------------ 2D context parallelism (Ulysses x ring)
class OracleRingOps(OracleOps):
    """The oracle's pieces plus attention with the rows' log-sum-exp and the merge."""

    def attention_lse(self, q, k, v, heads):
        B, m, Dh = q.shape
        dh = Dh // heads
        n = k.shape[1]
        qa = q.numpy().reshape(B, m, heads, dh)
        ka, va = k.numpy().reshape(B, n, heads, dh), v.numpy().reshape(B, n, heads, dh)
        o = np.stack([O.attention(qa[b], ka[b], va[b]).reshape(m, Dh) for b in range(B)])
        s = np.einsum("bmhd,bnhd->bhmn", qa, ka) / np.sqrt(dh) / np.log(2.0)   # log2 units
        mx = s.max(axis=-1, keepdims=True)
        lse = (mx + np.log2(np.exp2(s - mx).sum(axis=-1, keepdims=True)))[..., 0]
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge_state(self, q, heads):
        B, m, Dh = q.shape
        return torch.zeros((B, m, Dh), dtype=torch.float64), torch.zeros((B, heads, m), dtype=torch.float64)

    def merge(self, o_run, lse_run, o_part, lse_part, first, out=None):
        B, m, Dh = o_part.shape
        heads = lse_part.shape[1]
        if first:
            o_run.copy_(o_part)
            lse_run.copy_(lse_part)
        else:
            M = torch.maximum(lse_run, lse_part)
            a, c = torch.exp2(lse_run - M), torch.exp2(lse_part - M)
            wa = (a / (a + c)).permute(0, 2, 1).repeat_interleave(Dh // heads, dim=2)
            wc = (c / (a + c)).permute(0, 2, 1).repeat_interleave(Dh // heads, dim=2)
            o_run.copy_(wa * o_run + wc * o_part)
            lse_run.copy_(M + torch.log2(a + c))
        if out is not None:
            out.copy_(o_run)


@pytest.mark.parametrize("U,R", [(1, 2), (2, 2), (1, 4), (4, 1), (2, 1)])
def test_cp2d_in_one_process_equals_the_whole_block(U, R):
    d, w, kv, X, e0 = tiny_case()
    want = O.block_forward(X, e0, w, 0, kv, d)
    ops = OracleRingOps(d, w, kv, e0)
    blocks = [SP.CP2DBlock(ops, r, U, R, d.L, d.heads) for r in range(U * R)]
    X_locals = [torch.from_numpy(X[:, b.tok0:b.tok0 + b.n].copy()) for b in blocks]
    SP.cp2d_block_in_one_process(blocks, X_locals, 0)
    np.testing.assert_allclose(torch.cat(X_locals, dim=1).numpy(), want, atol=1e-10, rtol=0)


def test_ring_merge_by_log_sum_exp_is_the_attention_over_all_keys():
    rng = np.random.default_rng(9)
    q = torch.from_numpy(rng.standard_normal((2, 5, 8)))
    k, v = torch.from_numpy(rng.standard_normal((2, 12, 8))), torch.from_numpy(rng.standard_normal((2, 12, 8)))
    ops = OracleRingOps(None, None, None, None)
    o_all, lse_all = ops.attention_lse(q, k, v, 2)
    st = ops.merge_state(q, 2)
    for j, sl in enumerate([slice(0, 3), slice(3, 10), slice(10, 12)]):
        o, lse = ops.attention_lse(q, k[:, sl].contiguous(), v[:, sl].contiguous(), 2)
        ops.merge(st[0], st[1], o, lse, j == 0)
    np.testing.assert_allclose(st[0].numpy(), o_all.numpy(), atol=1e-12)
    np.testing.assert_allclose(st[1].numpy(), lse_all.numpy(), atol=1e-12)


def _cp2d_rank(rank, U, R, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=U * R, timeout=datetime.timedelta(seconds=60))
    try:
        d, w, kv, X, e0 = tiny_case()
        ul, rg = SP.cp2d_groups(U, R)
        blk = SP.CP2DBlock(OracleRingOps(d, w, kv, e0), rank, U, R, d.L, d.heads)
        X_local = torch.from_numpy(X[:, blk.tok0:blk.tok0 + blk.n].copy())
        blk.forward(0, X_local, SP.nccl_exchange(ul[blk.g]), SP.ring_pass_fn(rank, U, R))
        out[rank] = X_local.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("U,R", [(1, 2), (2, 2)])
def test_cp2d_gloo_ranks_equal_the_whole_block(U, R):
    d, w, kv, X, e0 = tiny_case()
    want = O.block_forward(X, e0, w, 0, kv, d)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_cp2d_rank, args=(r, U, R, port, out)) for r in range(U * R)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        got = np.concatenate([out[r] for r in range(U * R)], axis=1)
    np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)
