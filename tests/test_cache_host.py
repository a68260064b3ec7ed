"""The samplers' caches in model.py (host code) against the oracle's rules, on
the CPU ("Wan（通义万相）..." 5.3: CFG cache, attention cache, both at once;
7.2: the timestep MoE's choice of expert).
The library calls are replaced by recorders, so only the decision and
bookkeeping code of model.CfgCache, model.AttnCache and model.DiffusionCache
runs; the oracle's samplers run with a stand-in DiT (zeros) so that their own
per-step decisions can be read off.  Step counts and thresholds reach past
the 4-step schedules of the GPU sampler tests."""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from flow_matching_video_b200 import model, synth

WL = synth.TINY
SHAPE = (16, WL.dims.T, WL.dims.H, WL.dims.W)


class _Net:
    """A DiT stand-in that records its forwards."""

    def __init__(self, batch):
        self.batch, self.calls = batch, 0

    def forward(self, x, y, tau, stream=None):
        self.calls += 1
        return torch.zeros((self.batch,) + SHAPE)


def _oracle_decisions(monkeypatch, which, steps, **kw):
    d = WL.dims

    def fake_dit(xb, y, tau, w, kvs, dims, rnd=False, attn=None, **k):
        if attn is not None and not attn["reuse"]:
            for i in range(dims.blocks):
                attn["o"][i] = np.zeros((xb.shape[0], d.L, d.D))
        return np.zeros((xb.shape[0],) + SHAPE)
    monkeypatch.setattr(O, "dit_forward", fake_dit)
    w = synth.model_weights(WL)
    x = synth.inputs(WL)
    args = (x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, steps, 5.0)
    if which == "cfg":
        return O.sample_cfg_cache(*args, t_cfg=kw["t_cfg"])[2]
    if which == "attn":
        return O.sample_attn_cache(*args, t_attn=kw["t_attn"], interval=kw["interval"])[2]
    return O.sample_diffusion_cache(*args, t_cfg=kw["t_cfg"], t_attn=kw["t_attn"], interval=kw["interval"])[1]


def _cfg_cache(t_cfg):
    cc = model.CfgCache.__new__(model.CfgCache)
    cc.pair, cc.cond, cc.t_cfg = _Net(2), _Net(1), t_cfg
    cc.v_u, cc.have_v_u = torch.zeros(SHAPE), False
    return cc


def _attn_cache(t_attn, interval, net):
    ac = model.AttnCache.__new__(model.AttnCache)
    ac.net, ac.t_attn, ac.interval = net, t_attn, interval
    ac.o, ac.qkv = None, torch.zeros((2, 1))   # buffers: only sliced here, the recorders never read them
    ac.step, ac.last_fresh = 0, None
    return ac


@pytest.fixture
def no_library(monkeypatch):
    """The Euler update and the block-level forward replaced by recorders."""
    calls = []

    def fake_forward(net, x_t, y, tau, o, qkv, fresh, stream=None):
        calls.append((net.batch, fresh))
        return torch.zeros((net.batch,) + SHAPE)
    monkeypatch.setattr(model.wd, "wd_euler_cfg_step", lambda *a, **k: None)
    monkeypatch.setattr(model, "forward_reusing_attention", fake_forward)
    return calls


@pytest.mark.parametrize("steps,t_cfg", [(4, 0.5), (12, 0.5), (12, 0.0), (12, 1.0), (9, 0.35), (1, 0.5)])
def test_cfg_cache_runs_both_rows_when_the_oracle_does(monkeypatch, no_library, steps, t_cfg):
    cc = _cfg_cache(t_cfg)
    xb = torch.zeros((2,) + SHAPE)
    got = []
    for _, dt, tau in O.schedule(steps):
        before = cc.pair.calls
        cc.cfg_euler_step(xb, None, tau, dt, 5.0)
        got.append(cc.pair.calls > before)
    assert cc.pair.calls + cc.cond.calls == steps
    assert got == _oracle_decisions(monkeypatch, "cfg", steps, t_cfg=t_cfg)


@pytest.mark.parametrize("steps,t_attn,interval", [(4, 0.6, 2), (12, 0.5, 2), (12, 0.5, 3), (12, 0.0, 2),
                                                    (12, 1.0, 5), (10, 0.45, 1), (1, 0.5, 2)])
def test_attention_cache_recomputes_when_the_oracle_does(monkeypatch, no_library, steps, t_attn, interval):
    ac = _attn_cache(t_attn, interval, _Net(2))
    xb = torch.zeros((2,) + SHAPE)
    for _, dt, tau in O.schedule(steps):
        ac.cfg_euler_step(xb, None, tau, dt, 5.0)
    got = [f for _, f in no_library]
    assert got == _oracle_decisions(monkeypatch, "attn", steps, t_attn=t_attn, interval=interval)


@pytest.mark.parametrize("steps,t_cfg,t_attn,interval", [(12, 0.5, 0.5, 2), (12, 0.7, 0.3, 3), (12, 0.2, 0.8, 2),
                                                          (8, 0.5, 1.0, 4), (6, 1.0, 0.0, 2)])
def test_diffusion_cache_takes_the_oracle_decisions(monkeypatch, no_library, steps, t_cfg, t_attn, interval):
    dc = model.DiffusionCache.__new__(model.DiffusionCache)
    dc.cfg = _cfg_cache(t_cfg)
    dc.attn = _attn_cache(t_attn, interval, dc.cfg.pair)
    dc.o_cond = None
    xb = torch.zeros((2,) + SHAPE)
    for _, dt, tau in O.schedule(steps):
        dc.cfg_euler_step(xb, None, tau, dt, 5.0)
    got = [(batch == 2, fresh) for batch, fresh in no_library]
    assert got == _oracle_decisions(monkeypatch, "diffusion", steps, t_cfg=t_cfg, t_attn=t_attn, interval=interval)


class _Expert:
    def __init__(self):
        self.steps = 0

    def cfg_euler_step(self, xb, y, tau, dt, cfg_scale, stream=None):
        self.steps += 1
        return xb


@pytest.mark.parametrize("steps,t_moe", [(4, 0.6), (12, 0.5), (12, 0.875), (12, 1.0), (12, -1.0), (7, 0.4)])
def test_moe_runs_the_expert_the_oracle_picks(monkeypatch, steps, t_moe):
    moe = model.MoE.__new__(model.MoE)
    moe.high, moe.low, moe.t_moe = _Expert(), _Expert(), t_moe
    xb = torch.zeros((2,) + SHAPE)
    got = []
    for _, dt, tau in O.schedule(steps):
        before = moe.high.steps
        moe.cfg_euler_step(xb, None, tau, dt, 5.0)
        got.append("high" if moe.high.steps > before else "low")
    monkeypatch.setattr(O, "dit_forward", lambda xb, *a, **k: np.zeros((xb.shape[0],) + SHAPE))
    w = synth.model_weights(WL)
    x = synth.inputs(WL)
    used = O.sample_moe(x["x0"], x["img_lat"], w, w, x["txt"], x["clip"], WL.dims, steps, 5.0, t_moe)[2]
    assert got == used
