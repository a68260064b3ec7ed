"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own
independent problem; the step time is the max over ranks and the throughput
sums every rank's tokens.  No GPU needed."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, ms_by_rank, tokens, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, value = bench.reduce_over_ranks(ms_by_rank[rank], tokens, world)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_summed_tokens():
    world, tokens = 2, 1_965_600.0          # 2 x 32760 x 30 block-tokens per rank
    ms_by_rank = [500.0, 620.0]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, ms_by_rank, tokens, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        for r in range(world):
            ms, value = out[r]
            assert ms == 620.0                                   # slowest rank decides
            assert value == pytest.approx(world * tokens / 0.620)


def test_single_rank_is_local():
    import bench
    ms, value = bench.reduce_over_ranks(400.0, 1000.0, 1)
    assert ms == 400.0 and value == pytest.approx(2500.0)


# ------------------------------------------------------------------ CFG split over two ranks
class _StandInModel:
    """A deterministic batch-1 velocity field for the exchange test: the text
    row and the zeroed-text row differ, as the DiT's do."""

    def __init__(self, text_row: bool):
        self.text_row = text_row

    def forward(self, x1, y, tau):
        import torch
        base = torch.sin(x1 * 1.7 + tau / 1000.0)
        return base + (0.3 * torch.cos(x1) if self.text_row else 0.0)


def _euler(x, v_c, v_u, s, dt):
    x += dt * (v_u + s * (v_c - v_u))


def _cfg_rank(rank, world, port, x0, steps, out):
    import torch
    import torch.distributed as dist
    from flow_matching_video_b200.cfg_split import CfgSplit
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        split = CfgSplit(_StandInModel(text_row=(rank == 0)), euler=_euler)
        x = x0.clone()
        for k in range(steps):
            split.cfg_euler_step(x, None, 1000.0 * (1 - k / steps), 1.0 / steps, 5.0)
        out[rank] = x.numpy()
    finally:
        dist.destroy_process_group()


def test_cfg_split_two_gloo_ranks_match_the_single_process_step():
    import numpy as np
    import torch
    steps = 3
    x0 = torch.randn(16, 2, 4, 6, dtype=torch.float64, generator=torch.Generator().manual_seed(3))
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_cfg_rank, args=(r, 2, port, x0, steps, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        x0_, x1_ = out[0], out[1]
    # both ranks hold the same latent ...
    np.testing.assert_array_equal(x0_, x1_)
    # ... equal to the CFG Euler steps taken in one process with both rows
    cond, uncond = _StandInModel(True), _StandInModel(False)
    x = x0.clone()
    for k in range(steps):
        tau = 1000.0 * (1 - k / steps)
        _euler(x, cond.forward(x[None], None, tau)[0], uncond.forward(x[None], None, tau)[0], 5.0, 1.0 / steps)
    np.testing.assert_allclose(x0_, x.numpy(), rtol=0, atol=1e-15)


# ------------------------------------------------------------------ CFG split driving the real model orchestration
_COMPUTE = ("wd_build_cond_y", "wd_context_embed", "wd_cross_kv", "wd_time_mod", "wd_patch_embed",
            "wd_block_forward", "wd_unpatchify", "wd_euler_cfg_step")


def _cfg_dit_rank(rank, world, port, out):
    """One rank of the CFG split with a batch-1 model.DiT of the tiny model on
    the CPU: the library's compute calls are answered by the oracle (the
    stand-in of tests/fake_libwd.py); model.DiT, its context preparation and
    CfgSplit (all-gather of v, the CFG Euler update through the library's
    entry point) run as they do on GPUs."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from oracle import wan_oracle as O
    from flow_matching_video_b200 import model, synth, wd
    from flow_matching_video_b200.cfg_split import CfgSplit
    from fake_libwd import FakeWd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.TINY
        d = wl.dims
        w = synth.model_weights(wl)
        x = synth.inputs(wl)
        fake = FakeWd(wd, w, d)
        for name in _COMPUTE:            # this process only: the binding answers from the oracle
            setattr(wd, name, getattr(fake, name))
        dw = model.weights_to_device(w, d, "cpu")
        fake.bind(dw)
        net = model.DiT(d, dw, 1, device="cpu")
        txt = x["txt"] if rank == 0 else np.zeros_like(x["txt"])   # rank 1: the unconditional row
        net.prepare_context(torch.from_numpy(txt[None]), torch.from_numpy(x["clip"]))
        y = net.build_cond_y(torch.from_numpy(x["img_lat"]))
        split = CfgSplit(net)
        xx = torch.from_numpy(x["x0"]).clone()
        for t, dt, tau in O.schedule(wl.steps):
            split.cfg_euler_step(xx, y, tau, dt, wl.cfg_scale)
        out[rank] = (xx.numpy().astype(np.float64), [s.copy() for s in fake.seen_txt])
    finally:
        dist.destroy_process_group()


def test_cfg_split_two_gloo_ranks_with_the_model_equal_the_oracle_sampler():
    import numpy as np
    from oracle import wan_oracle as O
    from flow_matching_video_b200 import synth
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_cfg_dit_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        (x0_, txt0), (x1_, txt1) = out[0], out[1]
    wl = synth.TINY
    x = synth.inputs(wl)
    # rank 0's model saw the text, rank 1's zeroed text ("图解 Wan2.1 I2V" Q5)
    assert len(txt0) == len(txt1) == 1
    np.testing.assert_array_equal(txt0[0][0], x["txt"])
    assert not np.any(txt1[0])
    # both ranks hold the same latent, the oracle's 2-row CFG sampler
    np.testing.assert_array_equal(x0_, x1_)
    want, _ = O.sample(x["x0"], x["img_lat"], synth.model_weights(wl), x["txt"], x["clip"], wl.dims, wl.steps,
                       wl.cfg_scale)
    assert np.abs(x0_ - want).max() / np.sqrt((want ** 2).mean()) < 1e-5
    assert np.abs(want - x["x0"]).max() > 0.1


def _one_rank_split(port, out):
    import torch.distributed as dist
    from flow_matching_video_b200.cfg_split import CfgSplit
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        CfgSplit(object())
        out[0] = "accepted"
    except ValueError as e:
        out[0] = str(e)
    finally:
        dist.destroy_process_group()


def test_cfg_split_refuses_a_world_other_than_two():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        p = ctx.Process(target=_one_rank_split, args=(_free_port(), out))
        p.start()
        p.join(timeout=120)
        assert p.exitcode == 0 and "exactly two ranks" in out[0]


def test_bench_refuses_a_launcher_with_the_wrong_rank_count():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "--nproc-per-node 2" in r.stderr
