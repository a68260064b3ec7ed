"""More pins of the CPU oracle: the pieces of a block and of the sampler that
the other pin file checks only with a branch switched off.

* the token grid against the Conv3d output grid ("图解 Wan2.1 I2V" 5.1);
* the self-attention branch of a block with several tokens: adaLN, the fused
  projection, QK-RMSNorm over the full width D, the head split, 3D RoPE as a
  complex rotation per segment with positions from the token grid, and
  softmax attention — restated with torch (float64) and compared with the
  oracle ("图解 Wan2.1 I2V" 5.2, 5.3 (1) and (2));
* the cross-attention keys: each stream's keys come from its own weights
  (zero image key weights make the image stream the mean of its values),
  "图解 Wan2.1 I2V" 5.4;
* the text MLP and the CLIP MLPProj against torch ("图解 Wan2.1 I2V" 7);
* the sampler's unconditional row: zeroed text, CLIP and y unchanged
  ("图解 Wan2.1 I2V" Q5);
* the whole block with every branch on, against a torch restatement that runs
  self-attention, cross-attention and feed-forward one after the other
  ("图解 Wan2.1 I2V" 5.2-5.5), and the whole two-block model against a torch
  restatement of time MLP, patch embedding, context, blocks and head, and the
  three-step CFG Euler sampler around it.

Each pin is also run against oracles with a plausible mistake planted
(monkeypatched on the CPU, for the length of one test): the token grid with
rows and columns swapped, RMSNorm per head instead of over D, a RoPE turning
the wrong way or reading the wrong coordinate, the text and image key weights
swapped, the unconditional row keeping its text, the block's branches all
reading its input, every block running with block 0's weights, the guidance
combination with its rows exchanged.  The pin must fail on each.
"""
import unittest.mock as um

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

from oracle import wan_oracle as O
from flow_matching_video_b200 import synth

RNG = np.random.default_rng(11)


def T64(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def _tiny(T=2, H=4, W=6, D=48, heads=2, ffn=40, seed=99):
    """A tiny fp64 model whose token grid has T, H/2 and W/2 all different
    (2 x 2 x 3), so a swapped axis changes the positions."""
    d = synth.Dims(D=D, heads=heads, ffn=ffn, blocks=1, T=T, H=H, W=W, n_txt=5, c_txt=12,
                   n_img=4, c_img=10, dtype="f32")
    wl = synth.Workload("pin", d, batch=2, seed=seed)
    w = {k: v.astype(np.float64) for k, v in synth.model_weights(wl).items()}
    for k in list(w):                      # larger weights so that every term matters
        if k.endswith(".w"):
            w[k] = w[k] * 10
    txt = RNG.standard_normal((2, d.n_txt, d.c_txt))
    clip = RNG.standard_normal((d.n_img, d.c_img))
    X = RNG.standard_normal((2, d.L, D))
    return d, w, txt, clip, X


def _gated(w, D, g1, g2):
    """e0 and block weights such that gate1 = g1, gate2 = g2 exactly."""
    e0 = RNG.standard_normal((6, D))
    mod = w["blk0.mod"].copy()
    mod[2] = g1 - e0[2]
    mod[5] = g2 - e0[5]
    return e0, dict(w, **{"blk0.mod": mod})


# ------------------------------------------------------------------ token grid
def conv3d_token_grid(T, H, W):
    """(frame, row, column) of every token, read off a torch Conv3d with the
    patch embedding's kernel and stride (1, 2, 2) whose input channels carry
    each voxel's own coordinates; the tokens are the flattened output grid
    ("图解 Wan2.1 I2V" 5.1)."""
    f, yy, xx = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    x_in = T64(np.stack([f, yy, xx]))[None]                # [1, 3, T, H, W]
    wgt = torch.zeros(3, 3, 1, 2, 2, dtype=torch.float64)
    for c in range(3):
        wgt[c, c, 0, 0, 0] = 1.0                           # each patch's top-left voxel
    out = TF.conv3d(x_in, wgt, stride=(1, 2, 2))           # [1, 3, T, H/2, W/2]
    tok = out.flatten(2)[0].T.numpy()                      # [L, 3] in token order
    return tok[:, 0].astype(int), (tok[:, 1] // 2).astype(int), (tok[:, 2] // 2).astype(int)


def _grid_mismatch(T, H, W):
    want = conv3d_token_grid(T, H, W)
    got = O.grid_positions(T, H // 2, W // 2)
    return sum(int(np.any(np.asarray(g) != np.asarray(wv))) for g, wv in zip(got, want))


def test_grid_positions_are_the_conv3d_output_grid():
    for T, H, W in [(2, 4, 6), (3, 10, 14), (1, 2, 8), (5, 6, 4)]:
        assert _grid_mismatch(T, H, W) == 0
    # the same map as unravelling the token index over (T, H/2, W/2)
    f, y, x = np.unravel_index(np.arange(3 * 5 * 7), (3, 5, 7))
    np.testing.assert_array_equal(np.stack(O.grid_positions(3, 5, 7)), np.stack([f, y, x]))


def test_grid_pin_catches_swapped_rows_and_columns(monkeypatch):
    orig = O.grid_positions

    def swapped(T, Hp, Wp):   # rows and columns exchanged
        f, y, x = orig(T, Wp, Hp)
        return f, x, y
    monkeypatch.setattr(O, "grid_positions", swapped)
    assert _grid_mismatch(2, 4, 6) > 0


# ------------------------------------------------------------------ self-attention branch
def rope_complex(x, pos, dh):
    """3D RoPE as complex multiplication ("图解 Wan2.1 I2V" 5.3 (2)): each head
    of x [B, L, h, dh] is cut into frame / row / column segments of
    dh - 4(dh//6), 2(dh//6), 2(dh//6) channels; in segment s the channel pairs
    (2j, 2j+1) form the complex number z_j, multiplied by
    exp(i * p_s * 10000^(-2j/d_s)) with p_s the token's coordinate on axis s."""
    sizes = (dh - 4 * (dh // 6), 2 * (dh // 6), 2 * (dh // 6))
    out, off = [], 0
    for size, p in zip(sizes, pos):
        seg = x[..., off:off + size]
        z = torch.view_as_complex(seg.reshape(*seg.shape[:-1], size // 2, 2).contiguous())
        j = torch.arange(size // 2, dtype=torch.float64)
        theta = T64(p)[:, None] * torch.pow(torch.tensor(10000.0, dtype=torch.float64), -2.0 * j / size)
        rot = torch.polar(torch.ones_like(theta), theta)[None, :, None, :]   # [1, L, 1, size/2]
        out.append(torch.view_as_real(z * rot).reshape(seg.shape))
        off += size
    return torch.cat(out, dim=-1)


def self_branch_torch(X, e0, w, d, blk=0):
    """X + gate1 * Linear_o(attention) of one block, restated with torch:
    h = LayerNorm(X)(1 + scale1) + shift1; [q k v] = Linear_qkv(h);
    q, k = RMSNorm over D with gains; heads split; RoPE; SDPA; Linear_o."""
    B, L, D, h, dh = X.shape[0], d.L, d.D, d.heads, d.dh
    p = f"blk{blk}."
    mod = e0 + w[p + "mod"]
    Xt = T64(X)
    hh = TF.layer_norm(Xt, (D,), eps=d.eps) * (1 + T64(mod[1])) + T64(mod[0])
    q, k, v = TF.linear(hh, T64(w[p + "qkv.w"]), T64(w[p + "qkv.b"])).split(D, dim=-1)
    q = TF.rms_norm(q, (D,), weight=T64(w[p + "gq"]), eps=d.eps)
    k = TF.rms_norm(k, (D,), weight=T64(w[p + "gk"]), eps=d.eps)
    pos = conv3d_token_grid(d.T, d.H, d.W)
    heads = lambda t: t.reshape(B, L, h, dh)
    q, k, v = rope_complex(heads(q), pos, dh), rope_complex(heads(k), pos, dh), heads(v)
    o = TF.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2))
    o = o.transpose(1, 2).reshape(B, L, D)
    return (Xt + T64(mod[2]) * TF.linear(o, T64(w[p + "o.w"]), T64(w[p + "o.b"]))).numpy()


def _self_branch_error():
    d, w, txt, clip, X = _tiny()
    e0, w = _gated(w, d.D, 0.8, 0.0)
    # cross-attention output projection zero: the block is X + the self-attention branch
    w = dict(w, **{"blk0.co.w": np.zeros_like(w["blk0.co.w"]), "blk0.co.b": np.zeros(d.D)})
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv = O.cross_kv(w, 0, ctx_t, ctx_i)
    got = O.block_forward(X, e0, w, 0, kv, d)
    want = self_branch_torch(X, e0, w, d)
    # the branch moves X by far more than the comparison's bound
    assert np.abs(want - X).max() > 1.0
    return float(np.abs(got - want).max())


def test_block_self_attention_branch_against_torch_restatement():
    assert _self_branch_error() < 1e-10


def test_self_attention_pin_catches_swapped_grid_axes(monkeypatch):
    orig = O.grid_positions

    def swapped(T, Hp, Wp):
        f, y, x = orig(T, Wp, Hp)
        return f, x, y
    monkeypatch.setattr(O, "grid_positions", swapped)
    assert _self_branch_error() > 1e-3


def test_self_attention_pin_catches_rms_norm_per_head(monkeypatch):
    def per_head(x, eps, gamma=None, dh=24):   # the tiny model's head width
        x = np.asarray(x, np.float64)
        s = x.reshape(*x.shape[:-1], -1, dh)
        y = (s / np.sqrt((s * s).mean(axis=-1, keepdims=True) + eps)).reshape(x.shape)
        return y * gamma if gamma is not None else y
    monkeypatch.setattr(O, "rms_norm", per_head)
    assert _self_branch_error() > 1e-3


def test_self_attention_pin_catches_rope_turning_the_wrong_way(monkeypatch):
    orig = O.rope_3d
    monkeypatch.setattr(O, "rope_3d", lambda x, pf, py, px: orig(x, -np.asarray(pf), -np.asarray(py), -np.asarray(px)))
    assert _self_branch_error() > 1e-3


def test_self_attention_pin_catches_rope_reading_the_wrong_coordinate(monkeypatch):
    orig = O.rope_3d
    monkeypatch.setattr(O, "rope_3d", lambda x, pf, py, px: orig(x, pf, px, py))
    assert _self_branch_error() > 1e-3


def test_self_attention_pin_catches_rope_on_values(monkeypatch):
    # the oracle's branch with RoPE also applied to v: attention of (q, k, R v)
    orig_att = O.attention
    d = _tiny()[0]
    pf, py, px = conv3d_token_grid(d.T, d.H, d.W)

    def att(q, k, v):
        if v.shape[0] == d.L:   # self-attention (cross keys are fewer than L here)
            v = O.rope_3d(v, pf, py, px)
        return orig_att(q, k, v)
    monkeypatch.setattr(O, "attention", att)
    assert _self_branch_error() > 1e-3


# ------------------------------------------------------------------ the whole block, every branch on
def block_torch(X, e0, w, d, kv, blk=0):
    """One block with all three branches on, restated with torch (float64):
    the self-attention branch (self_branch_torch); then, on the stream it
    leaves, the decoupled cross-attention (affine LayerNorm, query Linear, the
    image and the text attention summed, output Linear; no adaLN, no gate);
    then, on the stream after that, the gated GELU feed-forward with adaLN
    ("图解 Wan2.1 I2V" 5.2-5.5)."""
    B, D, h, dh = X.shape[0], d.D, d.heads, d.dh
    p = f"blk{blk}."
    mod = e0 + w[p + "mod"]
    x1 = T64(self_branch_torch(X, e0, w, d, blk))
    hc = TF.layer_norm(x1, (D,), T64(w[p + "cn.g"]), T64(w[p + "cn.b"]), eps=d.eps)
    qc = TF.linear(hc, T64(w[p + "cq.w"]), T64(w[p + "cq.b"]))
    sp = lambda t: t.reshape(t.shape[0], t.shape[1], h, dh).transpose(1, 2)

    def sdpa(q, k, v):
        return TF.scaled_dot_product_attention(sp(q), sp(k), sp(v)).transpose(1, 2).reshape(q.shape)
    oc = sdpa(qc, T64(kv["k_txt"]), T64(kv["v_txt"]))
    if "k_img" in kv:   # the image-to-video model's second stream
        ki, vi = T64(kv["k_img"]).expand(B, -1, -1), T64(kv["v_img"]).expand(B, -1, -1)
        oc = sdpa(qc, ki, vi) + oc
    x2 = x1 + TF.linear(oc, T64(w[p + "co.w"]), T64(w[p + "co.b"]))
    h2 = TF.layer_norm(x2, (D,), eps=d.eps) * (1 + T64(mod[4])) + T64(mod[3])
    u = TF.gelu(TF.linear(h2, T64(w[p + "f1.w"]), T64(w[p + "f1.b"])))
    return (x2 + T64(mod[5]) * TF.linear(u, T64(w[p + "f2.w"]), T64(w[p + "f2.b"]))).numpy()


def _whole_block_error():
    d, w, txt, clip, X = _tiny()
    e0, w = _gated(w, d.D, 0.8, 1.3)
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv = O.cross_kv(w, 0, ctx_t, ctx_i)
    got = O.block_forward(X, e0, w, 0, kv, d)
    want = block_torch(X, e0, w, d, kv)
    assert np.abs(want - X).max() > 1.0
    return float(np.abs(got - want).max())


def test_whole_block_against_torch_restatement():
    assert _whole_block_error() < 1e-9


def test_whole_block_pin_catches_branches_reading_the_block_input(monkeypatch):
    """A plausible misreading of the order: the cross-attention and the
    feed-forward both read the block's input instead of the stream the branch
    before them left."""
    def parallel(Xr, o, e0, w, blk, kv, dims, rnd=False, fp8=False):
        p = f"blk{blk}."
        D, nh, dh, eps = dims.D, dims.heads, dims.dh, dims.eps
        _, _, gate1, shift2, scale2, gate2 = O._mod(e0, w, blk)
        sp = lambda a: np.asarray(a).reshape(-1, nh, dh)
        out = np.empty_like(np.asarray(Xr, np.float64))
        for b in range(Xr.shape[0]):
            x0 = Xr[b]
            sa = gate1 * O.linear(o[b], w[p + "o.w"], w[p + "o.b"])
            qc = sp(O.linear(O.layer_norm(x0, eps, w[p + "cn.g"], w[p + "cn.b"]), w[p + "cq.w"], w[p + "cq.b"]))
            oc = (O.attention(qc, sp(kv["k_img"]), sp(kv["v_img"]))
                  + O.attention(qc, sp(kv["k_txt"][b]), sp(kv["v_txt"][b]))).reshape(-1, D)
            ca = O.linear(oc, w[p + "co.w"], w[p + "co.b"])
            h2 = O.adaln_modulate(x0, shift2, scale2, eps, dims.norm)
            ff = gate2 * O.linear(O.gelu(O.linear(h2, w[p + "f1.w"], w[p + "f1.b"])), w[p + "f2.w"], w[p + "f2.b"])
            out[b] = x0 + sa + ca + ff
        return out
    monkeypatch.setattr(O, "block_after_attention", parallel)
    assert _whole_block_error() > 1e-3


# ------------------------------------------------------------------ the whole model
def dit_torch(x_t, y, tau, w, txt, clip, d):
    """The DiT's velocity restated with torch (float64): the time MLP on the
    sinusoid of tau ([cos, sin] at 10000^(-i/128)) giving e and the six
    modulation rows e0; the patch embedding as a Conv3d of concat(x_t, y); the
    text MLP and CLIP MLPProj; per block its cross keys and values and
    block_torch; the head (LayerNorm modulated by e + its own two rows, a
    Linear) and the inverse of the (1, 2, 2) patchify
    ("图解 Wan2.1 I2V" 4.2, 5.1-5.5, 7)."""
    W = lambda k: T64(w[k])
    B, D, T, Hp, Wp = x_t.shape[0], d.D, d.T, d.Hp, d.Wp
    fr = torch.pow(torch.tensor(10000.0, dtype=torch.float64), -torch.arange(128, dtype=torch.float64) / 128)
    es = torch.cat([torch.cos(tau * fr), torch.sin(tau * fr)])
    e = TF.linear(TF.silu(TF.linear(es, W("t1.w"), W("t1.b"))), W("t2.w"), W("t2.b"))
    e0 = TF.linear(TF.silu(e), W("tp.w"), W("tp.b")).reshape(6, D)
    x_in = T64(x_t) if y is None else torch.cat([T64(x_t), T64(y)[None].expand(B, -1, -1, -1, -1)], dim=1)
    X = TF.conv3d(x_in, W("pe.w").reshape(D, x_in.shape[1], 1, 2, 2), W("pe.b"), stride=(1, 2, 2))
    X = X.flatten(2).transpose(1, 2)
    mlp = lambda x, a, b: TF.linear(TF.gelu(TF.linear(x, W(a + ".w"), W(a + ".b"))), W(b + ".w"), W(b + ".b"))
    ctx_t = mlp(T64(txt), "txt1", "txt2")
    streams = [("k_txt", ctx_t, "ck"), ("v_txt", ctx_t, "cv")]
    if clip is not None:   # image-to-video: the CLIP context and its own keys and values
        ctx_i = mlp(T64(clip), "img1", "img2")
        streams += [("k_img", ctx_i, "cki"), ("v_img", ctx_i, "cvi")]
    for i in range(d.blocks):
        p = f"blk{i}."
        kv = {n: TF.linear(c, W(p + k + ".w"), W(p + k + ".b")).numpy() for n, c, k in streams}
        X = T64(block_torch(X.numpy(), e0.numpy(), w, d, kv, i))
    z = TF.layer_norm(X, (D,), eps=d.eps) * (1 + e + W("head.mod")[1]) + e + W("head.mod")[0]
    pt = TF.linear(z, W("head.w"), W("head.b"))                                   # [B, L, 16 * 1 * 2 * 2]
    return pt.reshape(B, T, Hp, Wp, 16, 2, 2).permute(0, 4, 1, 2, 5, 3, 6).reshape(B, 16, T, 2 * Hp, 2 * Wp).numpy()


def _whole_model_error(t2v=False):
    n_img, c_img = (0, 0) if t2v else (4, 10)
    d = synth.Dims(D=48, heads=2, ffn=40, blocks=2, T=2, H=4, W=6, n_txt=5, c_txt=12, n_img=n_img, c_img=c_img,
                   dtype="f32")
    wl = synth.Workload("pin2", d, batch=2, seed=98)
    w = {k: v.astype(np.float64) for k, v in synth.model_weights(wl).items()}
    for k in list(w):                      # larger weights so that every term matters
        if k.endswith(".w"):
            w[k] = w[k] * 6
    x_t = RNG.standard_normal((2, 16, d.T, d.H, d.W))
    y = None if t2v else RNG.standard_normal((20, d.T, d.H, d.W))
    txt = RNG.standard_normal((2, d.n_txt, d.c_txt))
    clip = None if t2v else RNG.standard_normal((d.n_img, d.c_img))
    tau = 731.0
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kvs = [O.cross_kv(w, i, ctx_t, ctx_i) for i in range(d.blocks)]
    got = O.dit_forward(x_t, y, tau, w, kvs, d)
    want = dit_torch(x_t, y, tau, w, txt, clip, d)
    assert np.abs(want).max() > 1.0
    return float(np.abs(got - want).max() / np.abs(want).max())


@pytest.mark.parametrize("t2v", [False, True])
def test_whole_model_against_torch_restatement(t2v):
    """Image-to-video, and text-to-video (x_t alone through a 16-channel patch
    embedding, text-only cross-attention; "图解 Wan2.1 I2V" 9)."""
    assert _whole_model_error(t2v) < 1e-12


def test_whole_model_pin_catches_every_block_reading_block_0(monkeypatch):
    """A dropped index: every block runs with block 0's weights (and its own
    cross keys and values)."""
    orig = O.block_forward
    monkeypatch.setattr(O, "block_forward", lambda X, e0, w, blk, kv, dims, *a, **k: orig(X, e0, w, 0, kv, dims, *a, **k))
    assert _whole_model_error() > 1e-3


def sample_torch(x0, img_lat, w, txt, clip, d, steps, s):
    """The CFG Euler sampler restated around dit_torch: y = the 4-channel mask
    (all ones on latent frame 0, the default known first frame) stacked on the
    image latent; the conditional row with the text, the unconditional row with
    zeroed text (CLIP and y kept); at step k of N, tau = 1000 (1 - k/N) and
    x += (1/N) (v_u + s (v_c - v_u)) ("图解 Wan2.1 I2V" 4.1, 7, Q5;
    "Wan（通义万相）..." 2.7)."""
    mask = np.zeros((4,) + img_lat.shape[1:])
    mask[:, 0] = 1.0
    y = np.concatenate([mask, img_lat])
    txt2 = np.stack([txt, np.zeros_like(txt)])
    x = np.asarray(x0, np.float64)
    for k in range(steps):
        v = dit_torch(np.stack([x, x]), y, 1000.0 * (1.0 - k / steps), w, txt2, clip, d)
        x = x + (1.0 / steps) * (v[1] + s * (v[0] - v[1]))
    return x


def _sampler_error():
    d = synth.Dims(D=48, heads=2, ffn=40, blocks=2, T=2, H=4, W=6, n_txt=5, c_txt=12, n_img=4, c_img=10,
                   dtype="f32")
    wl = synth.Workload("pin3", d, batch=2, seed=97)
    w = {k: v.astype(np.float64) for k, v in synth.model_weights(wl).items()}
    for k in list(w):
        if k.endswith(".w"):
            w[k] = w[k] * 6
    x0 = RNG.standard_normal((16, d.T, d.H, d.W))
    img_lat = RNG.standard_normal((16, d.T, d.H, d.W))
    txt = RNG.standard_normal((d.n_txt, d.c_txt))
    clip = RNG.standard_normal((d.n_img, d.c_img))
    got, _ = O.sample(x0, img_lat, w, txt, clip, d, steps=3, cfg_scale=5.0)
    want = sample_torch(x0, img_lat, w, txt, clip, d, 3, 5.0)
    assert np.abs(want - x0).max() > 1.0
    return float(np.abs(got - want).max() / np.abs(want).max())


def test_sampler_against_torch_restatement():
    assert _sampler_error() < 1e-12


def test_sampler_pin_catches_swapped_guidance_rows(monkeypatch):
    """The guidance combination with its rows exchanged (v_c + s (v_u - v_c))."""
    monkeypatch.setattr(O, "cfg_combine", lambda v_c, v_u, s: np.asarray(v_c) + s * (np.asarray(v_u) - np.asarray(v_c)))
    assert _sampler_error() > 1e-3


# ------------------------------------------------------------------ cross-attention keys and values
def _cross_setup():
    d, w, txt, clip, X = _tiny()
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    qc = RNG.standard_normal((7, d.heads, d.dh)) * 3
    return d, w, ctx_t, ctx_i, qc


def _cross_kv_errors(cross_kv):
    """With the image key weight zero, every image key is the bias, so the
    image stream of every query is the mean of the image values (and the text
    keys are unchanged); with the text key weight zero the text stream is the
    mean of the text values.  Returns the largest deviation."""
    d, w, ctx_t, ctx_i, qc = _cross_setup()
    nh, dh = d.heads, d.dh
    sp = lambda a: np.asarray(a).reshape(-1, nh, dh)
    errs = []
    full = cross_kv(w, 0, ctx_t, ctx_i)
    # the text keys and values of the full weights against torch
    kt = TF.linear(T64(ctx_t), T64(w["blk0.ck.w"]), T64(w["blk0.ck.b"])).numpy()
    vi = TF.linear(T64(ctx_i), T64(w["blk0.cvi.w"]), T64(w["blk0.cvi.b"])).numpy()
    errs += [np.abs(full["k_txt"] - kt).max(), np.abs(full["v_img"] - vi).max()]
    wz = dict(w, **{"blk0.cki.w": np.zeros_like(w["blk0.cki.w"])})
    z = cross_kv(wz, 0, ctx_t, ctx_i)
    o_img = O.attention(qc, sp(z["k_img"]), sp(z["v_img"]))
    errs.append(np.abs(o_img - sp(z["v_img"]).mean(axis=0)[None]).max())
    errs.append(np.abs(z["k_txt"] - full["k_txt"]).max())
    wz = dict(w, **{"blk0.ck.w": np.zeros_like(w["blk0.ck.w"])})
    z = cross_kv(wz, 0, ctx_t, ctx_i)
    o_txt = O.attention(qc, sp(z["k_txt"][0]), sp(z["v_txt"][0]))
    errs.append(np.abs(o_txt - sp(z["v_txt"][0]).mean(axis=0)[None]).max())
    errs.append(np.abs(z["k_img"] - full["k_img"]).max())
    return float(max(errs))


def test_cross_kv_each_stream_keys_from_its_own_weights():
    assert _cross_kv_errors(O.cross_kv) < 1e-10


def test_cross_kv_pin_catches_swapped_key_weights():
    def swapped(w, blk, ctx_txt, ctx_img, rnd=False):
        p = f"blk{blk}."
        w2 = dict(w, **{p + "ck.w": w[p + "cki.w"], p + "ck.b": w[p + "cki.b"],
                        p + "cki.w": w[p + "ck.w"], p + "cki.b": w[p + "ck.b"]})
        return O.cross_kv(w2, blk, ctx_txt, ctx_img, rnd)
    assert _cross_kv_errors(swapped) > 1e-3


# ------------------------------------------------------------------ context MLPs
def test_text_and_clip_mlps_against_torch():
    d, w, txt, clip, _ = _tiny()
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    mlp = lambda x, a, b: TF.linear(TF.gelu(TF.linear(T64(x), T64(w[a + ".w"]), T64(w[a + ".b"]))),
                                    T64(w[b + ".w"]), T64(w[b + ".b"])).numpy()
    np.testing.assert_allclose(ctx_t, mlp(txt, "txt1", "txt2"), atol=1e-11)
    np.testing.assert_allclose(ctx_i, mlp(clip, "img1", "img2"), atol=1e-11)
    assert ctx_i.shape == (d.n_img, d.D) and ctx_t.shape == (2, d.n_txt, d.D)


# ------------------------------------------------------------------ the sampler's two rows
def _sampler_inputs_seen(monkeypatch):
    """Run the tiny sampler and record what the context MLPs and the DiT see."""
    wl = synth.TINY
    d = wl.dims
    w = synth.model_weights(wl)
    x = synth.inputs(wl)
    seen = {"ctx": [], "fwd": []}
    orig_ctx, orig_fwd = O.context_embed, O.dit_forward

    def ctx(w_, txt, clip, rnd=False):
        seen["ctx"].append((np.array(txt), None if clip is None else np.array(clip)))
        return orig_ctx(w_, txt, clip, rnd)

    def fwd(x_t, y, tau, w_, kvs, dims, rnd=False):
        seen["fwd"].append((np.array(x_t), None if y is None else np.array(y)))
        return orig_fwd(x_t, y, tau, w_, kvs, dims, rnd)
    monkeypatch.setattr(O, "context_embed", ctx)
    monkeypatch.setattr(O, "dit_forward", fwd)
    O.sample(x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps, wl.cfg_scale)
    return x, seen


def _unconditional_row_ok(x, seen):
    (txt2, clip), = seen["ctx"]
    y_want = O.build_cond_y(x["img_lat"])
    ok = txt2.shape[0] == 2 and np.array_equal(txt2[0], x["txt"]) and not np.any(txt2[1])
    ok &= np.array_equal(clip, x["clip"])              # CLIP is kept for the unconditional row
    for xb, y in seen["fwd"]:
        ok &= xb.shape[0] == 2 and np.array_equal(xb[0], xb[1])   # both rows see the same latent
        ok &= y is not None and np.array_equal(y, y_want)          # and the same y
    return bool(ok) and len(seen["fwd"]) == synth.TINY.steps


def test_sampler_unconditional_row_zeroes_only_the_text(monkeypatch):
    x, seen = _sampler_inputs_seen(monkeypatch)
    assert np.any(x["txt"])
    assert _unconditional_row_ok(x, seen)


def test_unconditional_row_pin_catches_a_row_that_keeps_its_text(monkeypatch):
    orig_stack = np.stack
    txt_shape = synth.inputs(synth.TINY)["txt"].shape

    def keep_text(arrs, *a, **k):     # sample() builds [txt, 0]; plant [txt, txt]
        arrs = list(arrs)
        if len(arrs) == 2 and np.shape(arrs[0]) == txt_shape and not np.any(arrs[1]):
            arrs[1] = arrs[0]
        return orig_stack(arrs, *a, **k)
    monkeypatch.setattr(O.np, "stack", keep_text)
    x, seen = _sampler_inputs_seen(monkeypatch)
    assert not _unconditional_row_ok(x, seen)


# ------------------------------------------------------------------ attention cache ("Wan（通义万相）..." 5.3)
def test_attention_cache_decisions():
    # noise levels 1, 0.75, 0.5, 0.25 of a 4-step schedule
    levels = [1.0, 0.75, 0.5, 0.25]

    def pattern(t_attn, interval):
        last, out = None, []
        for k, lv in enumerate(levels):
            f = O.attn_cache_fresh(k, lv, last, t_attn, interval)
            last = k if f else last
            out.append(f)
        return out
    assert pattern(0.6, 2) == [True, True, False, True]
    assert pattern(0.6, 1) == [True] * 4           # interval 1 never reuses
    assert pattern(0.0, 3) == [True] * 4           # every noise level above 0: always recompute
    assert pattern(1.0, 4) == [True, False, False, False]


def test_attention_cache_never_taken_is_the_plain_sampler():
    wl = synth.TINY_MOE                            # the tiny model, 4 steps
    d, w, x = wl.dims, synth.model_weights(wl), synth.inputs(wl)
    want, trace = O.sample(x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps, wl.cfg_scale)
    got, trace2, fresh = O.sample_attn_cache(x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps,
                                             wl.cfg_scale, t_attn=0.6, interval=1)
    assert fresh == [True] * 4
    np.testing.assert_array_equal(got, want)


def test_attention_cache_reuse_is_exact_at_the_step_that_filled_it():
    """A forward that reuses the stored attention outputs at the same latent
    and noise level as the forward that stored them gives the same velocity;
    at another latent it differs from a fresh forward (the cache is used)."""
    d, w, txt, clip, X = _tiny()
    d = synth.Dims(**{**d.__dict__, "blocks": 1})
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kvs = [O.cross_kv(w, 0, ctx_t, ctx_i)]
    img = RNG.standard_normal((16, d.T, d.H, d.W))
    y = O.build_cond_y(img)
    xt = RNG.standard_normal((2, 16, d.T, d.H, d.W))
    cache = {"o": [None], "reuse": False}
    v_fresh = O.dit_forward(xt, y, 600.0, w, kvs, d, attn=cache)
    np.testing.assert_array_equal(v_fresh, O.dit_forward(xt, y, 600.0, w, kvs, d))
    cache["reuse"] = True
    np.testing.assert_array_equal(O.dit_forward(xt, y, 600.0, w, kvs, d, attn=cache), v_fresh)
    xt2 = xt + RNG.standard_normal(xt.shape)
    assert np.abs(O.dit_forward(xt2, y, 600.0, w, kvs, d, attn=cache) - O.dit_forward(xt2, y, 600.0, w, kvs, d)).max() > 1e-3


def test_attention_cache_pin_catches_a_cache_that_is_never_read(monkeypatch):
    """Planted mistake: the reusing step recomputes anyway.  Then the 4-step
    sampler with reuse equals the plain sampler, which the real cache does not."""
    wl = synth.TINY_MOE
    d, w, x = wl.dims, synth.model_weights(wl), synth.inputs(wl)
    plain, _ = O.sample(x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps, wl.cfg_scale)
    real, _, fresh = O.sample_attn_cache(x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps, wl.cfg_scale,
                                         t_attn=0.6, interval=2)
    assert fresh == [True, True, False, True]
    assert np.abs(real - plain).max() > 1e-6
    orig = O.dit_forward
    monkeypatch.setattr(O, "dit_forward", lambda *a, attn=None, **k: orig(*a, **k))
    broken, _, _ = O.sample_attn_cache(x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps, wl.cfg_scale,
                                       t_attn=0.6, interval=2)
    np.testing.assert_array_equal(broken, plain)


def test_diffusion_cache_reduces_to_each_cache_alone():
    """Both caches at once: with the attention cache never taken it is the CFG
    cache; with the CFG cache never taken it is the attention cache."""
    wl = synth.TINY_MOE
    d, w, x = wl.dims, synth.model_weights(wl), synth.inputs(wl)
    args = (x["x0"], x["img_lat"], w, x["txt"], x["clip"], d, wl.steps, wl.cfg_scale)
    cfg_only, _, fresh_cfg = O.sample_cfg_cache(*args, 0.5)
    both, dec = O.sample_diffusion_cache(*args, 0.5, 0.6, 1)
    assert [b for b, _ in dec] == fresh_cfg == [True, True, False, False]
    np.testing.assert_array_equal(both, cfg_only)
    attn_only, _, fresh_attn = O.sample_attn_cache(*args, 0.6, 2)
    both, dec = O.sample_diffusion_cache(*args, -1.0, 0.6, 2)      # t_cfg < 0: both rows every step
    assert [f for _, f in dec] == fresh_attn == [True, True, False, True]
    np.testing.assert_array_equal(both, attn_only)
    # together: the conditional-only steps reuse the conditional row's stored outputs
    both, dec = O.sample_diffusion_cache(*args, 0.5, 0.6, 2)
    assert dec == [(True, True), (True, True), (False, False), (False, True)]
    assert np.abs(both - cfg_only).max() > 1e-6 and np.abs(both - attn_only).max() > 1e-6


# ------------------------------------------------------------------ the FP8 block ("Wan（通义万相）..." 5.3)
def _e4m3_grid_rows(rows, cols, rng):
    """Rows whose values are e4m3 values times a power of two, each row holding
    +-448 x its scale, so that per-row quantisation is lossless."""
    grid = np.unique(np.abs(O.e4m3(rng.standard_normal(4000) * 50)))
    v = rng.choice(grid, size=(rows, cols)) * rng.choice([-1.0, 1.0], size=(rows, cols))
    v[:, 0] = 448.0
    return v * np.exp2(rng.integers(-12, -2, size=(rows, 1)).astype(np.float64))


def test_linear_fp8_is_exact_on_representable_operands():
    rng = np.random.default_rng(21)
    x, w, b = _e4m3_grid_rows(9, 48, rng), _e4m3_grid_rows(16, 48, rng), rng.standard_normal(16)
    np.testing.assert_array_equal(O.linear_fp8(x, w, b), O.linear(x, w, b))
    # a planted mistake that drops the weight scales is caught
    qx, sx = O.quant_rows_e4m3(x)
    qw, sw = O.quant_rows_e4m3(w)
    assert np.abs(O.gemm_fp8(qx, sx, qw, np.ones_like(sw), b) - O.linear(x, w, b)).max() > 1.0


def test_fp8_block_is_the_block_within_e4m3_precision():
    """The FP8 block differs from the exact block by the e4m3 rounding of its
    GEMM inputs (half a step: 2^-4 relative per element), far less than the
    block's own contribution, and by more than float64 noise (the quantisation
    is really applied)."""
    d, w, txt, clip, X = _tiny(D=48, ffn=40)
    e0 = RNG.standard_normal((6, d.D)) * 0.3
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv = O.cross_kv(w, 0, ctx_t, ctx_i)
    exact = O.block_forward(X, e0, w, 0, kv, d)
    f8 = O.block_forward(X, e0, w, 0, kv, d, fp8=True)
    contrib = np.sqrt(((exact - X) ** 2).mean())
    err = np.abs(f8 - exact).max()
    assert 1e-6 * contrib < err < 0.25 * contrib


def test_fp8_block_without_fp8_ffn2_is_the_fp8_block_with_an_exact_last_layer():
    """fp8="no-ffn2" keeps only the FFN's second layer exact: planting the
    exact Linear into that one call of the full FP8 block gives it bit for
    bit, and it differs from both."""
    d, w, txt, clip, X = _tiny(D=48, ffn=40)
    e0 = RNG.standard_normal((6, d.D)) * 0.3
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv = O.cross_kv(w, 0, ctx_t, ctx_i)
    exact = O.block_forward(X, e0, w, 0, kv, d)
    f8 = O.block_forward(X, e0, w, 0, kv, d, fp8=True)
    part = O.block_forward(X, e0, w, 0, kv, d, fp8="no-ffn2")
    assert np.abs(part - f8).max() > 0 and np.abs(part - exact).max() > 0
    lin8 = O.linear_fp8
    with um.patch.object(O, "linear_fp8", lambda x, wt, b=None: O.linear(x, wt, b) if wt is w["blk0.f2.w"] else lin8(x, wt, b)):
        planted = O.block_forward(X, e0, w, 0, kv, d, fp8=True)
    np.testing.assert_array_equal(planted, part)
