"""A stand-in for libwd's compute entry points on the CPU, for tests of the
host-side orchestration (model.DiT, cfg_split) without a GPU.

Every compute call is answered by the oracle in float64 on host tensors; the
size queries and the dims struct still come from the real binding (they need
no GPU).  The stand-in finds a block's weights by the addresses in the
weight structs, so it must be bound to the model's host tensors first.  It
also records what each call received (the text of the context projection,
the rows of each forward) so that tests can check who saw what.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import wan_oracle as O


class FakeWd:
    def __init__(self, real_wd, w_host: dict, dims):
        self.real = real_wd
        self.w = {k: np.asarray(v, np.float64) for k, v in w_host.items()}
        self.dims = dims
        self.by_ptr = {}
        self.ctx = {}            # ctx buffer address -> (ctx_txt, ctx_img)
        self.kv = {}             # kv buffer address -> oracle K/V dict
        self.seen_txt = []
        # the real binding's host-only helpers and structs
        for name in ("make_dims", "wd_ctx_bytes", "wd_kv_bytes", "wd_workspace_bytes", "wd_time_weights",
                     "wd_ctx_weights", "wd_block_weights", "wd_head_weights", "BLOCK_FIELDS"):
            setattr(self, name, getattr(real_wd, name))

    def bind(self, device_weights: dict):
        self.by_ptr = {t.data_ptr(): k for k, t in device_weights.items()}

    def _blk(self, block_w) -> int:
        return int(self.by_ptr[block_w.qkv_w].split(".")[0][3:])

    @staticmethod
    def _np(t):
        return t.detach().cpu().numpy().astype(np.float64)

    # ---------------------------------------------------------------- the path
    def wd_build_cond_y(self, cd, img_lat, y, known_frames=None, stream=None):
        y.copy_(torch.from_numpy(O.build_cond_y(self._np(img_lat), known_frames or (0,))))

    def wd_context_embed(self, cd, w, txt, clip, batch, ctx, stream=None):
        t = self._np(txt)
        self.seen_txt.append(t.copy())
        self.ctx[ctx.data_ptr()] = O.context_embed(self.w, t, None if clip is None else self._np(clip))

    def wd_cross_kv(self, cd, block_w, ctx, batch, kv, stream=None):
        ct, ci = self.ctx[ctx.data_ptr()]
        self.kv[kv.data_ptr()] = O.cross_kv(self.w, self._blk(block_w), ct, ci)

    def wd_time_mod(self, cd, time_w, tau, e, e0, stream=None):
        ee, ee0 = O.time_mod(self.w, tau, self.dims.D)
        e.copy_(torch.from_numpy(ee))
        e0.copy_(torch.from_numpy(ee0))

    def wd_patch_embed(self, cd, x_t, y, w, b, batch, X, ws, stream=None):
        X.copy_(torch.from_numpy(O.patch_embed(self._np(x_t), None if y is None else self._np(y),
                                               self.w["pe.w"], self.w["pe.b"])))

    def wd_block_forward(self, cd, block_w, e0, kv, batch, X, ws, stream=None):
        out = O.block_forward(self._np(X), self._np(e0), self.w, self._blk(block_w), self.kv[kv.data_ptr()],
                              self.dims)
        X.copy_(torch.from_numpy(out))

    def wd_unpatchify(self, cd, head_w, e, batch, X, v, ws, stream=None):
        v.copy_(torch.from_numpy(O.head_unpatchify(self._np(X), self._np(e), self.w, self.dims)))

    def wd_euler_cfg_step(self, x, v_cond, v_uncond, cfg_scale, dt, n=None, stream=None):
        vu = None if v_uncond is None else self._np(v_uncond)
        x.copy_(torch.from_numpy(O.euler_cfg_step(self._np(x), self._np(v_cond), vu, cfg_scale, dt)))
