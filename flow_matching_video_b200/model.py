"""Device-side Wan2.1-style DiT built on the libwd C ABI.

Holds the weights and buffers in device memory (torch tensors) and sequences
the entry points of libwd for one denoising forward and one CFG Euler step
("图解 Wan2.1 I2V" section 7), for the image-to-video model and its
text-to-video counterpart (section 9 of that page: n_img = 0), and the
two-expert timestep MoE sampler of Wan2.2 ("Wan（通义万相）..." 7.2).  Every
arithmetic step runs in libwd's kernels; this module only allocates, fills
structs of pointers and calls.
"""
from __future__ import annotations

import numpy as np
import torch

from . import synth
from . import wd

MATRIX_SUFFIX = ".w"


def _tdtype(dims: synth.Dims):
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


def weights_to_device(w_host: dict, dims: synth.Dims, device) -> dict:
    """numpy weights from synth.model_weights -> device tensors (matrices in the
    storage type, everything else fp32).  Time-MLP matrices stay fp32."""
    out = {}
    for k, a in w_host.items():
        is_mat = k.endswith(MATRIX_SUFFIX) and not k.startswith(("t1.", "t2.", "tp."))
        dt = _tdtype(dims) if is_mat else torch.float32
        out[k] = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=dt)
    return out


def random_weights_on_device(wl: synth.Workload, device) -> dict:
    """Seeded N(0, 0.02) weights drawn directly on the device (large stacks)."""
    d, s = wl.dims, wl.seed
    td = _tdtype(d)
    D, F = d.D, d.ffn
    std = synth.WEIGHT_STD
    w = {}

    def g(name, shape, dt=torch.float32, mean=0.0):
        w[name] = synth.device_normal(shape, std, mean, s, name, device, dt)

    g("t1.w", (D, synth.T_EMB)); g("t1.b", (D,)); g("t2.w", (D, D)); g("t2.b", (D,))
    g("tp.w", (6 * D, D)); g("tp.b", (6 * D,))
    g("pe.w", (D, d.patch_k), td); g("pe.b", (D,))
    g("txt1.w", (D, d.c_txt), td); g("txt1.b", (D,)); g("txt2.w", (D, D), td); g("txt2.b", (D,))
    if not d.t2v:
        g("img1.w", (D, d.c_img), td); g("img1.b", (D,)); g("img2.w", (D, D), td); g("img2.b", (D,))
    for i in range(d.blocks):
        p = f"blk{i}."
        for nm, shp in (("qkv", (3 * D, D)), ("o", (D, D)), ("cq", (D, D)), ("ck", (D, D)), ("cv", (D, D)),
                        ("cki", (D, D)), ("cvi", (D, D)), ("co", (D, D)), ("f1", (F, D)), ("f2", (D, F))):
            if d.t2v and nm in ("cki", "cvi"):
                continue
            g(p + nm + ".w", shp, td)
            g(p + nm + ".b", (shp[0],))
        g(p + "gq", (D,), mean=1.0); g(p + "gk", (D,), mean=1.0)
        g(p + "cn.g", (D,), mean=1.0); g(p + "cn.b", (D,))
        g(p + "mod", (6, D))
    g("head.mod", (2, D)); g("head.w", (synth.OUT_P, D), td); g("head.b", (synth.OUT_P,))
    return w


class DiT:
    """The DiT of one workload on one device, with its buffers for `batch` rows."""

    def __init__(self, dims: synth.Dims, weights: dict, batch: int, device="cuda", buffers_from: "DiT" = None,
                 fp8: bool = False, fp8_ffn2: bool = True, fp8_attention: bool = False):
        """buffers_from: another DiT of the same dims and batch whose workspace,
        residual stream and output buffers this one shares (the experts of a
        timestep MoE run one at a time); the context and K/V cache stay per model.
        fp8: the blocks run wd_block_forward_fp8 ("Wan（通义万相）..." 5.3), with the six
        matrices of every block quantised once here by the library's row
        quantiser (per output channel); fp8_ffn2=False keeps the FFN's second
        layer in bf16 (its input, the FFN hidden, is then not quantised);
        fp8_attention: the self-attention as the page's FP8 attention (INT8
        Q K^T, FP8 P V)."""
        self.dims = dims
        self.cd = wd.make_dims(dims)
        self.batch = batch
        self.device = torch.device(device)
        self.w = weights
        self.tdtype = _tdtype(dims)
        p = lambda k: self.w[k].data_ptr() if k in self.w else 0   # image weights: none for text-to-video
        self.time_w = wd.wd_time_weights(*(p(k) for k in ("t1.w", "t1.b", "t2.w", "t2.b", "tp.w", "tp.b")))
        self.ctx_w = wd.wd_ctx_weights(*(p(k) for k in ("txt1.w", "txt1.b", "txt2.w", "txt2.b",
                                                        "img1.w", "img1.b", "img2.w", "img2.b")))
        names = {"qkv_w": "qkv.w", "qkv_b": "qkv.b", "g_q": "gq", "g_k": "gk", "o_w": "o.w", "o_b": "o.b",
                 "cn_g": "cn.g", "cn_b": "cn.b", "cq_w": "cq.w", "cq_b": "cq.b", "ck_w": "ck.w", "ck_b": "ck.b",
                 "cv_w": "cv.w", "cv_b": "cv.b", "cki_w": "cki.w", "cki_b": "cki.b", "cvi_w": "cvi.w",
                 "cvi_b": "cvi.b", "co_w": "co.w", "co_b": "co.b", "f1_w": "f1.w", "f1_b": "f1.b",
                 "f2_w": "f2.w", "f2_b": "f2.b", "mod": "mod"}
        self.block_w = [wd.wd_block_weights(*(p(f"blk{i}." + names[f]) for f in wd.BLOCK_FIELDS))
                        for i in range(dims.blocks)]
        self.head_w = wd.wd_head_weights(p("head.mod"), p("head.w"), p("head.b"))
        self.fp8 = fp8
        self.q8, self.block_w8 = {}, []
        if fp8:
            for i in range(dims.blocks):
                ptrs = {}
                for nm in ("qkv", "o", "cq", "co", "f1", "f2"):
                    if nm == "f2" and not fp8_ffn2:
                        ptrs["f2_q"] = ptrs["f2_s"] = None
                        continue
                    wt = self.w[f"blk{i}.{nm}.w"]
                    q = torch.empty(wt.shape, dtype=torch.uint8, device=wt.device)
                    sc = torch.empty(wt.shape[0], dtype=torch.float32, device=wt.device)
                    wd.wd_quant_rows_e4m3(wd.WD_BF16, wt.shape[0], wt.shape[1], wt, q, sc)
                    self.q8[(i, nm)] = (q, sc)
                    ptrs[nm + "_q"], ptrs[nm + "_s"] = q.data_ptr(), sc.data_ptr()
                self.block_w8.append(wd.wd_block_weights_fp8(*(ptrs[f] for f in wd.FP8_FIELDS),
                                                             int(bool(fp8_attention))))
        L, D = dims.L, dims.D
        dev = self.device
        self.ctx = torch.empty(wd.wd_ctx_bytes(self.cd, batch), dtype=torch.uint8, device=dev)
        kvb = wd.wd_kv_bytes(self.cd, batch)
        self.kv = torch.empty((dims.blocks, kvb), dtype=torch.uint8, device=dev)
        if buffers_from is not None:
            assert buffers_from.dims == dims and buffers_from.batch == batch
            src = buffers_from
            self.ws, self.X, self.e, self.e0, self.v = src.ws, src.X, src.e, src.e0, src.v
            return
        ws_bytes = wd.wd_workspace_bytes_fp8(self.cd, batch) if fp8 else wd.wd_workspace_bytes(self.cd, batch)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.X = torch.empty((batch, L, D), dtype=torch.float32, device=dev)
        self.e = torch.empty(D, dtype=torch.float32, device=dev)
        self.e0 = torch.empty((6, D), dtype=torch.float32, device=dev)
        self.v = torch.empty((batch, 16, dims.T, dims.H, dims.W), dtype=torch.float32, device=dev)

    # -------------------------------------------------------------- once per video
    def build_cond_y(self, img_lat: torch.Tensor, known_frames=None) -> torch.Tensor:
        y = torch.empty((20,) + tuple(img_lat.shape[1:]), dtype=torch.float32, device=self.device)
        wd.wd_build_cond_y(self.cd, img_lat, y, known_frames)
        return y

    def prepare_context(self, txt: torch.Tensor, clip: torch.Tensor = None):
        """txt [batch, n_txt, c_txt], clip [n_img, c_img] in the storage type
        (None for the text-to-video model)."""
        wd.wd_context_embed(self.cd, self.ctx_w, txt, clip, self.batch, self.ctx)
        for i in range(self.dims.blocks):
            wd.wd_cross_kv(self.cd, self.block_w[i], self.ctx, self.batch, self.kv[i])

    # -------------------------------------------------------------- per step
    def forward(self, x_t: torch.Tensor, y: torch.Tensor, tau: float, stream=None) -> torch.Tensor:
        """v = DiT(concat(x_t, y), tau) for x_t [batch, 16, T, H, W]; returns self.v.
        y is None for the text-to-video model."""
        wd.wd_time_mod(self.cd, self.time_w, tau, self.e, self.e0, stream)
        wd.wd_patch_embed(self.cd, x_t, y, self.w["pe.w"], self.w["pe.b"], self.batch, self.X, self.ws, stream)
        for i in range(self.dims.blocks):
            if self.fp8:
                wd.wd_block_forward_fp8(self.cd, self.block_w[i], self.block_w8[i], self.e0, self.kv[i], self.batch,
                                        self.X, self.ws, stream)
            else:
                wd.wd_block_forward(self.cd, self.block_w[i], self.e0, self.kv[i], self.batch, self.X, self.ws, stream)
        wd.wd_unpatchify(self.cd, self.head_w, self.e, self.batch, self.X, self.v, self.ws, stream)
        return self.v

    def cfg_euler_step(self, xb: torch.Tensor, y: torch.Tensor, tau: float, dt: float, cfg_scale: float,
                       stream=None):
        """One CFG Euler step on xb [2, 16, T, H, W] (both rows hold x; row 0
        sees the text, row 1 zeroed text): x += dt (v_u + s (v_c - v_u))."""
        assert self.batch == 2
        v = self.forward(xb, y, tau, stream)
        wd.wd_euler_cfg_step(xb[0], v[0], v[1], cfg_scale, dt, stream=stream)
        xb[1].copy_(xb[0])
        return xb


class MoE:
    """Timestep-level mixture of two experts of one architecture (Wan2.2,
    "Wan（通义万相）..." 7.2): every CFG Euler step runs the high-noise expert
    while the noise level tau / 1000 exceeds t_moe, the low-noise expert from
    there on.  The experts share their device buffers."""

    def __init__(self, dims: synth.Dims, w_high: dict, w_low: dict, t_moe: float, batch: int = 2, device="cuda"):
        self.high = DiT(dims, w_high, batch, device)
        self.low = DiT(dims, w_low, batch, device, buffers_from=self.high)
        self.t_moe = t_moe

    def prepare_context(self, txt: torch.Tensor, clip: torch.Tensor = None):
        self.high.prepare_context(txt, clip)
        self.low.prepare_context(txt, clip)

    def expert(self, tau: float) -> DiT:
        return self.high if tau / 1000.0 > self.t_moe else self.low

    def cfg_euler_step(self, xb: torch.Tensor, y: torch.Tensor, tau: float, dt: float, cfg_scale: float,
                       stream=None):
        return self.expert(tau).cfg_euler_step(xb, y, tau, dt, cfg_scale, stream)


class CfgCache:
    """CFG cache ("Wan（通义万相）..." 5.3, skip the unconditional path in the late
    steps): while the noise level tau / 1000 exceeds t_cfg a step evaluates both
    rows; from the first step at or below it only the conditional row runs
    (a batch-1 model on the same weights, with its own K/V cache of the
    conditional text) and the CFG combination reuses the last unconditional
    velocity computed."""

    def __init__(self, dims: synth.Dims, weights: dict, t_cfg: float, device="cuda"):
        self.pair = DiT(dims, weights, 2, device)
        self.cond = DiT(dims, weights, 1, device)
        self.t_cfg = t_cfg
        self.v_u = torch.empty((16, dims.T, dims.H, dims.W), dtype=torch.float32, device=self.pair.device)
        self.have_v_u = False

    def prepare_context(self, txt: torch.Tensor, clip: torch.Tensor = None):
        """txt [2, n_txt, c_txt] (row 0 the text, row 1 zeroed)."""
        self.pair.prepare_context(txt, clip)
        self.cond.prepare_context(txt[:1].contiguous(), clip)
        self.have_v_u = False

    def fresh(self, tau: float) -> bool:
        return not self.have_v_u or tau / 1000.0 > self.t_cfg

    def cfg_euler_step(self, xb: torch.Tensor, y: torch.Tensor, tau: float, dt: float, cfg_scale: float,
                       stream=None):
        """xb [2, 16, T, H, W] as for DiT.cfg_euler_step."""
        if self.fresh(tau):
            v = self.pair.forward(xb, y, tau, stream)
            self.v_u.copy_(v[1])
            self.have_v_u = True
            v_c = v[0]
        else:
            v_c = self.cond.forward(xb[:1], y, tau, stream)[0]
        wd.wd_euler_cfg_step(xb[0], v_c, self.v_u, cfg_scale, dt, stream=stream)
        xb[1].copy_(xb[0])
        return xb


def forward_reusing_attention(net: DiT, x_t, y, tau: float, o: torch.Tensor, qkv: torch.Tensor, fresh: bool,
                              stream=None) -> torch.Tensor:
    """A forward of `net` whose blocks either compute their self-attention
    output into o[i] (fresh) or take it from there: o [blocks, net.batch, L, D]
    and qkv [net.batch, L, 3D] in the storage type (qkv is scratch)."""
    d = net.dims
    wd.wd_time_mod(net.cd, net.time_w, tau, net.e, net.e0, stream)
    wd.wd_patch_embed(net.cd, x_t, y, net.w["pe.w"], net.w["pe.b"], net.batch, net.X, net.ws, stream)
    for i in range(d.blocks):
        if fresh:
            wd.wd_block_qkv(net.cd, net.block_w[i], net.e0, net.batch, 0, d.L, net.X, qkv, net.ws, stream)
            wd.wd_block_self_attention(net.cd, net.batch, d.heads, qkv, o[i], stream)
        wd.wd_block_post(net.cd, net.block_w[i], net.e0, net.kv[i], net.batch, d.L, o[i], net.X, net.ws, stream)
    wd.wd_unpatchify(net.cd, net.head_w, net.e, net.batch, net.X, net.v, net.ws, stream)
    return net.v


class AttnCache:
    """Attention cache ("Wan（通义万相）..." 5.3, reuse attention outputs across
    steps): each block's self-attention output o (the input of its output
    projection) is kept per block and batch row.  A step recomputes it while
    nothing is stored, while its noise level tau / 1000 exceeds t_attn, and
    otherwise once `interval` steps have passed since the last recomputation;
    the steps in between skip each block's norm, q/k/v projection, QK-norm,
    RoPE and self-attention and run only wd_block_post on the stored o.
    Memory: blocks x batch x L x D elements of the storage type (6 GB for the
    30-block 480p model at batch 2)."""

    def __init__(self, dims: synth.Dims, weights: dict, t_attn: float, interval: int, batch: int = 2,
                 device="cuda"):
        if interval < 1:
            raise ValueError("interval must be >= 1")
        self.net = DiT(dims, weights, batch, device)
        self.t_attn, self.interval = t_attn, interval
        net = self.net
        self.o = torch.empty((dims.blocks, batch, dims.L, dims.D), dtype=net.tdtype, device=net.device)
        self.qkv = torch.empty((batch, dims.L, 3 * dims.D), dtype=net.tdtype, device=net.device)
        self.step = 0
        self.last_fresh = None

    def prepare_context(self, txt: torch.Tensor, clip: torch.Tensor = None):
        self.net.prepare_context(txt, clip)
        self.step, self.last_fresh = 0, None

    def fresh(self, tau: float) -> bool:
        return (self.last_fresh is None or tau / 1000.0 > self.t_attn
                or self.step - self.last_fresh >= self.interval)

    def forward(self, x_t: torch.Tensor, y: torch.Tensor, tau: float, stream=None) -> torch.Tensor:
        """One forward; recomputes or reuses the attention outputs as fresh(tau) says."""
        fresh = self.fresh(tau)
        v = forward_reusing_attention(self.net, x_t, y, tau, self.o, self.qkv, fresh, stream)
        if fresh:
            self.last_fresh = self.step
        self.step += 1
        return v

    def cfg_euler_step(self, xb: torch.Tensor, y: torch.Tensor, tau: float, dt: float, cfg_scale: float,
                       stream=None):
        """xb [2, 16, T, H, W] as for DiT.cfg_euler_step."""
        v = self.forward(xb, y, tau, stream)
        wd.wd_euler_cfg_step(xb[0], v[0], v[1], cfg_scale, dt, stream=stream)
        xb[1].copy_(xb[0])
        return xb


class DiffusionCache:
    """The attention cache and the CFG cache together ("Wan（通义万相）..." 5.3,
    "diffusion cache"): while the noise level exceeds t_cfg both rows run
    (batch 2), afterwards the conditional row alone (batch 1) with the last
    unconditional velocity reused; in either case each block's self-attention
    output is recomputed or reused by the attention cache's rule (t_attn,
    interval; one step counter).  A conditional-only step reads and writes the
    conditional row's stored outputs."""

    def __init__(self, dims: synth.Dims, weights: dict, t_cfg: float, t_attn: float, interval: int, device="cuda"):
        self.cfg = CfgCache(dims, weights, t_cfg, device)
        self.attn = AttnCache.__new__(AttnCache)   # the rule and the buffers, on the pair model
        self.attn.net, self.attn.t_attn, self.attn.interval = self.cfg.pair, t_attn, interval
        net = self.cfg.pair
        self.attn.o = torch.empty((dims.blocks, 2, dims.L, dims.D), dtype=net.tdtype, device=net.device)
        self.attn.qkv = torch.empty((2, dims.L, 3 * dims.D), dtype=net.tdtype, device=net.device)
        self.attn.step, self.attn.last_fresh = 0, None
        # the conditional row's slices of the buffers (contiguous per block)
        self.o_cond = [self.attn.o[i, :1] for i in range(dims.blocks)]

    def prepare_context(self, txt: torch.Tensor, clip: torch.Tensor = None):
        self.cfg.prepare_context(txt, clip)
        self.attn.step, self.attn.last_fresh = 0, None

    def cfg_euler_step(self, xb: torch.Tensor, y: torch.Tensor, tau: float, dt: float, cfg_scale: float,
                       stream=None):
        """xb [2, 16, T, H, W] as for DiT.cfg_euler_step."""
        cc, ac = self.cfg, self.attn
        fresh = ac.fresh(tau)
        if cc.fresh(tau):
            v = forward_reusing_attention(cc.pair, xb, y, tau, ac.o, ac.qkv, fresh, stream)
            cc.v_u.copy_(v[1])
            cc.have_v_u = True
            v_c = v[0]
        else:
            v_c = forward_reusing_attention(cc.cond, xb[:1], y, tau, self.o_cond, ac.qkv[:1], fresh, stream)[0]
        if fresh:
            ac.last_fresh = ac.step
        ac.step += 1
        wd.wd_euler_cfg_step(xb[0], v_c, cc.v_u, cfg_scale, dt, stream=stream)
        xb[1].copy_(xb[0])
        return xb
