"""CFG split over two ranks: one video's CFG Euler step on two GPUs.

Classifier-free guidance needs two forwards per step, one with the text and
one with zeroed text ("图解 Wan2.1 I2V" section 7 and Q5).  They are
independent, so rank 0 evaluates the conditional row and rank 1 the
unconditional row, each with a batch-1 model; one all-gather of the velocity
(16 x T x H x W fp32, 8.4 MB at 480p/81 frames) is the only exchange per step.
Both ranks then apply the same CFG Euler update to their copy of the latent,
so the latent stays replicated without a broadcast.

This module is the host logic only: the forward and the update run in libwd
(a batch-1 `model.DiT`, `wd.wd_euler_cfg_step`); the exchange is
torch.distributed (NCCL between GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class CfgSplit:
    """net: this rank's batch-1 model, its context prepared with the text on
    rank 0 and with zeroed text on rank 1.  euler(x, v_c, v_u, s, dt) updates
    x in place (default: libwd's CFG Euler kernel)."""

    def __init__(self, net, group=None, euler=None):
        if dist.get_world_size(group) != 2:
            raise ValueError("the CFG split takes exactly two ranks")
        self.net = net
        self.group = group
        self.rank = dist.get_rank(group)
        if euler is None:
            from . import wd
            euler = lambda x, v_c, v_u, s, dt: wd.wd_euler_cfg_step(x, v_c, v_u, s, dt)
        self.euler = euler
        self._v = None

    def cfg_euler_step(self, x: torch.Tensor, y, tau: float, dt: float, cfg_scale: float) -> torch.Tensor:
        """x [16, T, H, W], identical on both ranks; returns it updated in place."""
        v = self.net.forward(x[None], y, tau)[0]
        if self._v is None or self._v[0].shape != v.shape:
            self._v = [torch.empty_like(v) for _ in range(2)]
        dist.all_gather(self._v, v.contiguous(), group=self.group)
        v_c, v_u = self._v   # rank 0 holds the text row, rank 1 the zeroed-text row
        self.euler(x, v_c, v_u, cfg_scale, dt)
        return x
