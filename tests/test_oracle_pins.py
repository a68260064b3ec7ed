"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test checks an oracle function against something other than itself: a
number the pages print (tests/golden/pages_numbers.json), a closed form, an
invariant, a special case that reduces to a library routine (torch, run in
float64), or brute force on tiny inputs.  No GPU is needed.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

from oracle import wan_oracle as O
from flow_matching_video_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))
RNG = np.random.default_rng(7)


def T64(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


# ------------------------------------------------------------------ rounding
def test_bf16_round_matches_torch_conversion():
    a = (RNG.standard_normal(20000) * np.exp(RNG.uniform(-20, 20, 20000))).astype(np.float32)
    # exact ties: low 16 bits = 0x8000, both parities of the kept bit
    u = RNG.integers(0x3F000000, 0x47000000, 4000, dtype=np.uint32)
    ties = ((u & 0xFFFF0000) | 0x8000).view(np.float32)
    a = np.concatenate([a, ties, -ties])
    want = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16(a), want)


def test_fp16_round_matches_numpy_half():
    # normals, subnormals (|a| < 2**-14), overflow to infinity (> 65504)
    a = RNG.standard_normal(20000) * np.exp(RNG.uniform(-25, 12, 20000))
    # exact ties halfway between neighbouring halves, both parities of the kept bit
    h = RNG.integers(1, 0x7BFF, 4000, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    ties = (lo + hi) / 2
    a = np.concatenate([a, ties, -ties, [0.0, -0.0, 65504.0, 65519.0, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26]])
    with np.errstate(over="ignore"):
        want = a.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(O.fp16(a), want)
    # ties go to the even neighbour
    even = np.where(h % 2 == 0, lo, hi)
    np.testing.assert_array_equal(O.fp16(ties), even)


# ------------------------------------------------------------------ shapes printed on the pages
def test_key_numbers():
    k = GOLD["key_numbers"]
    assert k["y_channels"] == k["mask_channels"] + k["latent_channels"]
    assert k["dit_in_channels_i2v"] == k["latent_channels"] + k["y_channels"] == synth.IN_C
    assert (k["clip_image_side"] // k["clip_patch_side"]) ** 2 + 1 == k["clip_tokens"]
    assert k["context_tokens"] == k["clip_tokens"] + k["text_tokens"]
    assert synth.PATCH_K == k["dit_in_channels_i2v"] * int(np.prod(k["patch"]))
    assert synth.T_EMB == k["time_embedding_width"]
    assert k["mask_channels"] == k["vae_temporal_stride"]


@pytest.mark.parametrize("case", GOLD["token_counts"]["cases"])
def test_token_count(case):
    assert O.token_count(case["F"], case["H"], case["W"]) == case["L"]
    assert 1 + (case["F"] - 1) // 4 == case["T_lat"]


def test_workload_token_counts():
    assert synth.BLOCK_480P17.dims.L == 7800
    assert synth.STACK_480P81.dims.L == 32760
    assert synth.WIDE_720P81.dims.L == 75600
    assert synth.TINY.dims.L == 32


@pytest.mark.parametrize("dh", [128, 32])
def test_rope_split_formula(dh):
    assert list(O.rope_split(dh)) == GOLD["rope_split_formula"][f"dh_{dh}"]
    assert sum(O.rope_split(dh)) == dh


# ------------------------------------------------------------------ mask and y
def test_mask_first_frame():
    m = O.mask_frames(21)
    assert m.shape == (4, 21)
    assert np.all(m[:, 0] == 1.0) and np.all(m[:, 1:] == 0.0)


def test_mask_known_frames_positions():
    T = 6
    F = 4 * (T - 1) + 1
    for p in range(1, F):
        m = O.mask_frames(T, known_pixel_frames=(p,))
        assert m.sum() == 1.0
        f, c = divmod(p + 3, 4)       # pixel frame p sits after the 4 copies of frame 0
        assert m[c, f] == 1.0
    # first and last frame known ([I2V] Q6): last pixel frame lands in channel 3 of the last latent frame
    m = O.mask_frames(T, (0, F - 1))
    assert np.all(m[:, 0] == 1) and m[3, T - 1] == 1 and m.sum() == 5


def test_build_cond_y_layout():
    img = RNG.standard_normal((16, 3, 4, 6))
    y = O.build_cond_y(img)
    assert y.shape == (20, 3, 4, 6)
    assert np.all(y[:4, 0] == 1) and np.all(y[:4, 1:] == 0)
    np.testing.assert_array_equal(y[4:], img)


# ------------------------------------------------------------------ elementwise
def test_silu_gelu_closed_forms_and_library():
    assert O.silu(0.0) == 0.0 and abs(O.silu(1.0) - 1 / (1 + math.exp(-1))) < 1e-15
    x = RNG.standard_normal(1000) * 4
    np.testing.assert_allclose(O.gelu(x), TF.gelu(T64(x), approximate="none").numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(O.silu(x), TF.silu(T64(x)).numpy(), rtol=0, atol=1e-14)
    assert O.gelu(0.0) == 0.0


def test_layer_norm_moments_and_library():
    x = RNG.standard_normal((50, 96)) * 3 + 1
    y = O.layer_norm(x, 0.0)
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    np.testing.assert_allclose((y * y).mean(-1), 1, atol=1e-12)
    g, b = RNG.standard_normal(96), RNG.standard_normal(96)
    want = TF.layer_norm(T64(x), (96,), T64(g), T64(b), eps=1e-6).numpy()
    np.testing.assert_allclose(O.layer_norm(x, 1e-6, g, b), want, atol=1e-12)


def test_rms_norm_library():
    x = RNG.standard_normal((50, 96)) * 3 + 1
    g = RNG.standard_normal(96)
    want = TF.rms_norm(T64(x), (96,), T64(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, 1e-6, g), want, atol=1e-12)
    np.testing.assert_allclose((O.rms_norm(x, 0.0) ** 2).mean(-1), 1, atol=1e-12)


def test_adaln_modulate_special_cases():
    x = RNG.standard_normal((10, 64))
    z = np.zeros(64)
    ln = O.layer_norm(x, 1e-6)
    np.testing.assert_array_equal(O.adaln_modulate(x, z, z, 1e-6), ln)
    np.testing.assert_allclose(O.adaln_modulate(x, z, np.ones(64), 1e-6), 2 * ln, atol=1e-14)
    c = RNG.standard_normal(64)
    np.testing.assert_allclose(O.adaln_modulate(x, c, z, 1e-6), ln + c, atol=1e-14)
    np.testing.assert_array_equal(O.adaln_modulate(x, z, z, 1e-6, "rms"), O.rms_norm(x, 1e-6))


# ------------------------------------------------------------------ timestep embedding
def test_sinusoid_closed_form():
    e = O.sinusoid(0.0)
    assert e.shape == (256,)
    np.testing.assert_array_equal(e[:128], 1.0)
    np.testing.assert_array_equal(e[128:], 0.0)
    tau = 437.5
    for i in (0, 1, 64, 127):
        w = 10000.0 ** (-i / 128)
        assert abs(O.sinusoid(tau)[i] - math.cos(tau * w)) < 1e-12
        assert abs(O.sinusoid(tau)[128 + i] - math.sin(tau * w)) < 1e-12


def test_time_mod_structure():
    D = 8
    w = {k: RNG.standard_normal(s) for k, s in
         (("t1.w", (D, 256)), ("t1.b", (D,)), ("t2.w", (D, D)), ("t2.b", (D,)),
          ("tp.w", (6 * D, D)), ("tp.b", (6 * D,)))}
    # zero first layer: e = W2 silu(b1) + b2, computed by hand with scalar loops
    w0 = dict(w, **{"t1.w": np.zeros((D, 256))})
    e, e0 = O.time_mod(w0, 123.0, D)
    for r in range(D):
        acc = w["t2.b"][r]
        for c in range(D):
            b1 = w["t1.b"][c]
            acc += w["t2.w"][r, c] * b1 / (1 + math.exp(-b1))
        assert abs(e[r] - acc) < 1e-12
    # zero projection: e0 is the projection bias cut into 6 consecutive chunks of D
    w1 = dict(w, **{"tp.w": np.zeros((6 * D, D))})
    _, e0 = O.time_mod(w1, 5.0, D)
    for k in range(6):
        np.testing.assert_array_equal(e0[k], w["tp.b"][k * D:(k + 1) * D])
    # the timestep enters only through the sinusoid
    e_a, _ = O.time_mod(w, 10.0, D)
    e_b, _ = O.time_mod(w, 900.0, D)
    assert np.abs(e_a - e_b).max() > 1e-3


# ------------------------------------------------------------------ RoPE
def _rope_input(N=7, h=2, dh=32):
    return RNG.standard_normal((N, h, dh))


def test_rope_identity_at_origin():
    x = _rope_input()
    z = np.zeros(x.shape[0])
    np.testing.assert_array_equal(O.rope_3d(x, z, z, z), x)


def test_rope_norm_preserving_per_pair():
    x = _rope_input()
    p = RNG.integers(0, 30, (3, x.shape[0]))
    y = O.rope_3d(x, *p)
    np.testing.assert_allclose(x[..., 0::2] ** 2 + x[..., 1::2] ** 2,
                               y[..., 0::2] ** 2 + y[..., 1::2] ** 2, atol=1e-12)


def test_rope_segments_follow_their_coordinate():
    dh = 32
    dT, dH, dW = O.rope_split(dh)
    x = _rope_input(N=1, h=1, dh=dh)
    base = O.rope_3d(x, [0], [0], [0])
    yf = O.rope_3d(x, [3], [0], [0])
    yy = O.rope_3d(x, [0], [3], [0])
    yx = O.rope_3d(x, [0], [0], [3])
    seg = [slice(0, dT), slice(dT, dT + dH), slice(dT + dH, dh)]
    for y, moved in ((yf, 0), (yy, 1), (yx, 2)):
        for s in range(3):
            changed = np.abs(y[..., seg[s]] - base[..., seg[s]]).max() > 1e-9
            assert changed == (s == moved)


def test_rope_pair_rotation_closed_form():
    dh = 128
    dT, dH, dW = O.rope_split(dh)
    for off, size, axis in ((0, dT, 0), (dT, dH, 1), (dT + dH, dW, 2)):
        for j in (0, 1, size // 2 - 1):
            x = np.zeros((1, 1, dh))
            x[0, 0, off + 2 * j] = 1.0
            pos = [[0], [0], [0]]
            pos[axis] = [5]
            y = O.rope_3d(x, *pos)
            th = 5 * 10000.0 ** (-2.0 * j / size)
            assert abs(y[0, 0, off + 2 * j] - math.cos(th)) < 1e-12
            assert abs(y[0, 0, off + 2 * j + 1] - math.sin(th)) < 1e-12


def test_rope_relative_position_property():
    dh = 32
    q, k = RNG.standard_normal((1, 1, dh)), RNG.standard_normal((1, 1, dh))

    def dot(pq, pk):
        return float((O.rope_3d(q, *[[v] for v in pq]) * O.rope_3d(k, *[[v] for v in pk])).sum())

    for _ in range(20):
        pq, pk, sh = RNG.integers(0, 40, 3), RNG.integers(0, 40, 3), RNG.integers(-10, 10, 3)
        assert abs(dot(pq, pk) - dot(pq + sh, pk + sh)) < 1e-10


# ------------------------------------------------------------------ attention
def test_attention_matches_library_sdpa():
    q, k, v = RNG.standard_normal((37, 3, 16)), RNG.standard_normal((53, 3, 16)), RNG.standard_normal((53, 3, 16))
    want = TF.scaled_dot_product_attention(T64(q).transpose(0, 1), T64(k).transpose(0, 1),
                                           T64(v).transpose(0, 1)).transpose(0, 1).numpy()
    np.testing.assert_allclose(O.attention(q, k, v), want, atol=1e-12)


def test_attention_brute_force_logsumexp():
    q, k, v = RNG.standard_normal((5, 2, 4)), RNG.standard_normal((6, 2, 4)), RNG.standard_normal((6, 2, 4))
    got = O.attention(q, k, v)
    for i in range(5):
        for h in range(2):
            s = [sum(q[i, h, d] * k[j, h, d] for d in range(4)) / 2.0 for j in range(6)]
            lse = math.log(sum(math.exp(x) for x in s))
            for d in range(4):
                assert abs(got[i, h, d] - sum(math.exp(s[j] - lse) * v[j, h, d] for j in range(6))) < 1e-12


def test_attention_degenerate_cases():
    q = RNG.standard_normal((9, 2, 8))
    k1, v1 = RNG.standard_normal((1, 2, 8)), RNG.standard_normal((1, 2, 8))
    np.testing.assert_allclose(O.attention(q, k1, v1), np.broadcast_to(v1, (9, 2, 8)), atol=1e-14)
    k = np.broadcast_to(k1, (11, 2, 8))
    v = RNG.standard_normal((11, 2, 8))
    np.testing.assert_allclose(O.attention(q, k, v), np.broadcast_to(v.mean(0), (9, 2, 8)), atol=1e-13)


# ------------------------------------------------------------------ patchify / unpatchify
def test_patch_embed_is_conv3d():
    B, T, H, W, D = 2, 3, 6, 8, 10
    x_t = RNG.standard_normal((B, 16, T, H, W))
    y = RNG.standard_normal((20, T, H, W))
    w = RNG.standard_normal((D, 36, 1, 2, 2))
    b = RNG.standard_normal(D)
    got = O.patch_embed(x_t, y, w.reshape(D, 144), b)               # [B, L, D]
    x_in = np.concatenate([x_t, np.broadcast_to(y, (B,) + y.shape)], axis=1)
    ref = TF.conv3d(T64(x_in), T64(w), T64(b), stride=(1, 2, 2)).numpy()   # [B, D, T, H/2, W/2]
    np.testing.assert_allclose(got, ref.reshape(B, D, -1).transpose(0, 2, 1), atol=1e-12)


def test_unpatchify_inverts_patchify_and_index_map():
    B, C, T, Hp, Wp = 2, 16, 3, 4, 5
    v = RNG.standard_normal((B, C, T, 2 * Hp, 2 * Wp))
    np.testing.assert_array_equal(O.unpatchify(O.patchify(v), T, Hp, Wp), v)
    p = RNG.standard_normal((B, T * Hp * Wp, 64))
    u = O.unpatchify(p, T, Hp, Wp)
    for (b, c, f, yy, xx, kh, kw) in [(0, 0, 0, 0, 0, 0, 0), (1, 15, 2, 3, 4, 1, 1), (0, 7, 1, 2, 3, 1, 0)]:
        l = (f * Hp + yy) * Wp + xx
        assert u[b, c, f, 2 * yy + kh, 2 * xx + kw] == p[b, l, c * 4 + kh * 2 + kw]


# ------------------------------------------------------------------ blocks
def _tiny(T=2, H=4, W=6, D=32, heads=2, ffn=48):
    d = synth.Dims(D=D, heads=heads, ffn=ffn, blocks=1, T=T, H=H, W=W, n_txt=5, c_txt=12,
                   n_img=3, c_img=10, dtype="f32")
    wl = synth.Workload("t", d, batch=2, seed=99)
    w = {k: v.astype(np.float64) for k, v in synth.model_weights(wl).items()}
    for k in list(w):                      # larger weights so every branch matters
        if k.endswith(".w"):
            w[k] = w[k] * 10
    txt = RNG.standard_normal((2, d.n_txt, d.c_txt))
    clip = RNG.standard_normal((d.n_img, d.c_img))
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv = O.cross_kv(w, 0, ctx_t, ctx_i)
    X = RNG.standard_normal((2, d.L, D))
    return d, w, kv, X


def _gates(w, D, g1, g2, rng_e0=True):
    e0 = RNG.standard_normal((6, D)) if rng_e0 else np.zeros((6, D))
    mod = w["blk0.mod"].copy()
    mod[2] = g1 - e0[2]
    mod[5] = g2 - e0[5]
    return e0, dict(w, **{"blk0.mod": mod})


def test_block_adaln_zero_identity():
    d, w, kv, X = _tiny()
    e0, w = _gates(w, d.D, 0.0, 0.0)
    w = dict(w, **{"blk0.co.w": np.zeros_like(w["blk0.co.w"]), "blk0.co.b": np.zeros(d.D)})
    np.testing.assert_array_equal(O.block_forward(X, e0, w, 0, kv, d), X)


def test_block_ffn_branch_against_library():
    d, w, kv, X = _tiny()
    e0, w = _gates(w, d.D, 0.0, 1.7)
    w = dict(w, **{"blk0.co.w": np.zeros_like(w["blk0.co.w"]), "blk0.co.b": np.zeros(d.D)})
    mod = e0 + w["blk0.mod"]
    h2 = TF.layer_norm(T64(X), (d.D,), eps=1e-6) * (1 + T64(mod[4])) + T64(mod[3])
    u = TF.gelu(TF.linear(h2, T64(w["blk0.f1.w"]), T64(w["blk0.f1.b"])))
    want = X + 1.7 * TF.linear(u, T64(w["blk0.f2.w"]), T64(w["blk0.f2.b"])).numpy()
    np.testing.assert_allclose(O.block_forward(X, e0, w, 0, kv, d), want, atol=1e-11)


def test_block_cross_branch_against_library():
    d, w, kv, X = _tiny()
    e0, w = _gates(w, d.D, 0.0, 0.0)
    hc = TF.layer_norm(T64(X), (d.D,), T64(w["blk0.cn.g"]), T64(w["blk0.cn.b"]), eps=1e-6)
    qc = TF.linear(hc, T64(w["blk0.cq.w"]), T64(w["blk0.cq.b"]))
    B, L, D, h, dh = 2, d.L, d.D, d.heads, d.dh

    def sdpa(q, k, v):   # q [B, L, D], k/v [B, N, D]
        sp = lambda t: t.reshape(t.shape[0], t.shape[1], h, dh).transpose(1, 2)
        return TF.scaled_dot_product_attention(sp(q), sp(k), sp(v)).transpose(1, 2).reshape(q.shape)

    kt, vt = T64(kv["k_txt"]), T64(kv["v_txt"])
    ki, vi = T64(kv["k_img"]).expand(B, -1, -1), T64(kv["v_img"]).expand(B, -1, -1)
    oc = sdpa(qc, ki, vi) + sdpa(qc, kt, vt)
    want = X + TF.linear(oc, T64(w["blk0.co.w"]), T64(w["blk0.co.b"])).numpy()
    np.testing.assert_allclose(O.block_forward(X, e0, w, 0, kv, d), want, atol=1e-11)


def test_block_self_attention_single_token_is_value_path():
    # one token: attention returns v, so the branch is Linear_o(Linear_v(h)) and RoPE does not matter
    d, w, kv, _ = _tiny(T=1, H=2, W=2)
    X = RNG.standard_normal((2, 1, d.D))
    e0, w = _gates(w, d.D, 0.9, 0.0)
    w = dict(w, **{"blk0.co.w": np.zeros_like(w["blk0.co.w"]), "blk0.co.b": np.zeros(d.D)})
    mod = e0 + w["blk0.mod"]
    h = TF.layer_norm(T64(X), (d.D,), eps=1e-6) * (1 + T64(mod[1])) + T64(mod[0])
    wv, bv = w["blk0.qkv.w"][2 * d.D:], w["blk0.qkv.b"][2 * d.D:]
    v = TF.linear(h, T64(wv), T64(bv))
    want = X + 0.9 * TF.linear(v, T64(w["blk0.o.w"]), T64(w["blk0.o.b"])).numpy()
    np.testing.assert_allclose(O.block_forward(X, e0, w, 0, kv, d), want, atol=1e-11)


def test_block_row_sampling_is_exact():
    d, w, kv, X = _tiny()
    e0 = RNG.standard_normal((6, d.D)) * 0.3
    full = O.block_forward(X, e0, w, 0, kv, d)
    rows = np.array([0, 5, d.L - 1])
    np.testing.assert_allclose(O.block_forward(X, e0, w, 0, kv, d, rows=rows), full[:, rows], atol=1e-12)


def test_dual_cross_attention_equal_streams_doubles():
    q = RNG.standard_normal((7, 2, 8))
    k, v = RNG.standard_normal((4, 2, 8)), RNG.standard_normal((4, 2, 8))
    np.testing.assert_allclose(O.attention(q, k, v) + O.attention(q, k, v), 2 * O.attention(q, k, v))


def test_context_zero_text_is_constant():
    d, w, _, _ = _tiny()
    ctx_t, _ = O.context_embed(w, np.zeros((1, d.n_txt, d.c_txt)), np.zeros((d.n_img, d.c_img)))
    want = O.gelu(w["txt1.b"]) @ w["txt2.w"].T + w["txt2.b"]
    np.testing.assert_allclose(ctx_t[0], np.broadcast_to(want, ctx_t[0].shape), atol=1e-13)


def test_head_unpatchify_index_map():
    d, w, _, _ = _tiny(D=64, heads=2, ffn=32)
    X = RNG.standard_normal((2, d.L, d.D))
    e = RNG.standard_normal(d.D)
    w = dict(w, **{"head.w": np.eye(64, d.D), "head.b": np.zeros(64)})
    v = O.head_unpatchify(X, e, w, d)
    z = O.layer_norm(X, 1e-6) * (1 + e + w["head.mod"][1]) + e + w["head.mod"][0]
    for (b, c, f, yy, xx, kh, kw) in [(0, 0, 0, 0, 0, 0, 0), (1, 15, 1, 1, 2, 1, 1), (0, 9, 0, 1, 0, 0, 1)]:
        l = (f * d.Hp + yy) * d.Wp + xx
        assert abs(v[b, c, f, 2 * yy + kh, 2 * xx + kw] - z[b, l, c * 4 + kh * 2 + kw]) < 1e-12


# ------------------------------------------------------------------ flow matching, Euler, CFG
def test_fm_path_endpoints_and_velocity():
    x0, x1 = RNG.standard_normal(50), RNG.standard_normal(50)
    np.testing.assert_array_equal(O.fm_path(x0, x1, 0.0), x0)
    np.testing.assert_array_equal(O.fm_path(x0, x1, 1.0), x1)
    hstep = 1e-6
    fd = (O.fm_path(x0, x1, 0.3 + hstep) - O.fm_path(x0, x1, 0.3 - hstep)) / (2 * hstep)
    np.testing.assert_allclose(fd, O.fm_velocity(x0, x1), atol=1e-8)


def test_euler_exact_velocity_lands_on_data():
    x0, x1 = RNG.standard_normal(100), RNG.standard_normal(100)
    v = O.fm_velocity(x0, x1)
    np.testing.assert_array_equal(O.euler_cfg_step(x0, v, None, 5.0, 1.0), x0 + v)
    np.testing.assert_allclose(O.euler_cfg_step(x0, v, None, 5.0, 1.0), x1, atol=1e-15)
    for N in (2, 7, 12):
        x, _ = O.sample(x0, None, None, None, None, None, N, 5.0, model=lambda x, tau: (v, v))
        np.testing.assert_allclose(x, x1, atol=1e-13)


def test_cfg_special_cases():
    vc, vu = RNG.standard_normal(30), RNG.standard_normal(30)
    np.testing.assert_allclose(O.cfg_combine(vc, vu, 1.0), vc, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(O.cfg_combine(vc, vu, 0.0), vu)
    for s in (0.0, 5.0, 7.5):
        np.testing.assert_allclose(O.cfg_combine(vc, vc, s), vc, atol=1e-15)
    np.testing.assert_allclose(O.cfg_combine(vc, vu, 5.0), vu + 5.0 * (vc - vu))


def test_schedule():
    for N in (1, 2, 12):
        s = O.schedule(N)
        assert len(s) == N and s[0][0] == 0.0 and abs(sum(d for _, d, _ in s) - 1.0) < 1e-15
        assert s[0][2] == 1000.0 and abs(s[-1][2] - 1000.0 / N) < 1e-9


def test_tiny_sampler_runs_and_guidance_matters():
    wl = synth.TINY
    w = synth.model_weights(wl)
    x = synth.inputs(wl)
    xf, trace = O.sample(x["x0"], x["img_lat"], w, x["txt"], x["clip"], wl.dims, wl.steps, wl.cfg_scale)
    assert xf.shape == (16, 2, 8, 8) and np.all(np.isfinite(xf))
    vc, vu = trace[0]
    assert np.abs(vc - vu).max() > 1e-6          # zeroed text changes the prediction
    np.testing.assert_allclose(xf, O.euler_cfg_step(O.euler_cfg_step(x["x0"], *trace[0], 5.0, 0.5),
                                                    *trace[1], 5.0, 0.5), atol=1e-14)


# ------------------------------------------------------------------ text-to-video model ([I2V] 9)
def test_t2v_patch_embed_is_conv3d_of_16_channels():
    B, T, H, W, D = 2, 3, 6, 8, 10
    x_t = RNG.standard_normal((B, 16, T, H, W))
    w = RNG.standard_normal((D, 16, 1, 2, 2))
    b = RNG.standard_normal(D)
    got = O.patch_embed(x_t, None, w.reshape(D, 64), b)
    ref = TF.conv3d(T64(x_t), T64(w), T64(b), stride=(1, 2, 2)).numpy()
    np.testing.assert_allclose(got, ref.reshape(B, D, -1).transpose(0, 2, 1), atol=1e-12)


def test_t2v_block_is_i2v_block_without_image_values():
    # with V_img = 0 the image stream adds nothing, so the dual cross-attention
    # of the image-to-video block reduces to the single text stream
    d, w, kv, X = _tiny()
    e0 = RNG.standard_normal((6, d.D))
    w = dict(w, **{"blk0.cvi.w": np.zeros_like(w["blk0.cvi.w"]), "blk0.cvi.b": np.zeros(d.D)})
    txt = RNG.standard_normal((2, d.n_txt, d.c_txt))
    clip = RNG.standard_normal((d.n_img, d.c_img))
    ctx_t, ctx_i = O.context_embed(w, txt, clip)
    kv_i2v = O.cross_kv(w, 0, ctx_t, ctx_i)
    assert np.all(kv_i2v["v_img"] == 0)
    kv_t2v = O.cross_kv(w, 0, ctx_t, None)
    assert set(kv_t2v) == {"k_txt", "v_txt"}
    np.testing.assert_allclose(O.block_forward(X, e0, w, 0, kv_t2v, d), O.block_forward(X, e0, w, 0, kv_i2v, d),
                               atol=1e-12)
    # ... and the image stream does matter when its values are not zero
    w2 = dict(w, **{"blk0.cvi.b": np.ones(d.D)})
    kv2 = O.cross_kv(w2, 0, ctx_t, ctx_i)
    assert np.abs(O.block_forward(X, e0, w2, 0, kv2, d) - O.block_forward(X, e0, w2, 0, kv_t2v, d)).max() > 1e-3


def test_t2v_context_has_no_clip_branch():
    w = synth.model_weights(synth.TINY_T2V)
    assert "img1.w" not in w and "blk0.cki.w" not in w and w["pe.w"].shape == (128, 64)
    txt = RNG.standard_normal((2, 16, 64))
    ctx_t, ctx_i = O.context_embed(w, txt, None)
    assert ctx_i is None and ctx_t.shape == (2, 16, 128)


def test_t2v_tiny_sampler_runs_and_guidance_matters():
    wl = synth.TINY_T2V
    w = synth.model_weights(wl)
    x = synth.inputs(wl)
    xf, trace = O.sample(x["x0"], None, w, x["txt"], None, wl.dims, wl.steps, wl.cfg_scale)
    assert xf.shape == (16, 2, 8, 8) and np.all(np.isfinite(xf))
    assert np.abs(trace[0][0] - trace[0][1]).max() > 1e-6


# ------------------------------------------------------------------ timestep MoE ([WAN] 7.2)
def test_moe_expert_choice_follows_noise_level():
    assert O.expert_for(1.0, 0.6) == "high" and O.expert_for(0.61, 0.6) == "high"
    assert O.expert_for(0.6, 0.6) == "low" and O.expert_for(0.25, 0.6) == "low"
    # on the 4-step grid the noise levels are 1, 0.75, 0.5, 0.25
    assert [O.expert_for(tau / 1000.0, 0.6) for _, _, tau in O.schedule(4)] == ["high", "high", "low", "low"]


def _moe_inputs():
    wl = synth.TINY_MOE
    w_hi, w_lo = (synth.model_weights(e) for e in synth.experts(wl))
    return wl, w_hi, w_lo, synth.inputs(wl)


def test_moe_with_one_expert_throughout_is_the_plain_sampler():
    wl, w_hi, w_lo, x = _moe_inputs()
    args = (x["txt"], x["clip"], wl.dims, wl.steps, wl.cfg_scale)
    x_lo, _, used = O.sample_moe(x["x0"], x["img_lat"], w_hi, w_lo, *args, t_moe=1.0)
    assert used == ["low"] * wl.steps
    np.testing.assert_array_equal(x_lo, O.sample(x["x0"], x["img_lat"], w_lo, *args)[0])
    x_hi, _, used = O.sample_moe(x["x0"], x["img_lat"], w_hi, w_lo, *args, t_moe=-1.0)
    assert used == ["high"] * wl.steps
    np.testing.assert_array_equal(x_hi, O.sample(x["x0"], x["img_lat"], w_hi, *args)[0])


def test_moe_with_identical_experts_is_the_plain_sampler_and_the_switch_matters():
    wl, w_hi, w_lo, x = _moe_inputs()
    args = (x["txt"], x["clip"], wl.dims, wl.steps, wl.cfg_scale)
    x_same, _, used = O.sample_moe(x["x0"], x["img_lat"], w_hi, w_hi, *args, t_moe=wl.t_moe)
    assert used == ["high", "high", "low", "low"]
    np.testing.assert_array_equal(x_same, O.sample(x["x0"], x["img_lat"], w_hi, *args)[0])
    x_moe, _, _ = O.sample_moe(x["x0"], x["img_lat"], w_hi, w_lo, *args, t_moe=wl.t_moe)
    assert np.abs(x_moe - x_same).max() > 1e-3


# ------------------------------------------------------------------ CFG cache ([WAN] 5.3)
def test_cfg_cache_never_taken_is_the_plain_sampler():
    wl = synth.TINY_MOE   # 4 steps: noise levels 1, 0.75, 0.5, 0.25
    w = synth.model_weights(wl)
    x = synth.inputs(wl)
    args = (x["txt"], x["clip"], wl.dims, wl.steps, wl.cfg_scale)
    xc, _, fresh = O.sample_cfg_cache(x["x0"], x["img_lat"], w, *args, t_cfg=0.0)
    assert fresh == [True] * 4
    np.testing.assert_array_equal(xc, O.sample(x["x0"], x["img_lat"], w, *args)[0])


def test_cfg_cache_reuses_the_last_unconditional_velocity():
    wl = synth.TINY_MOE
    w = synth.model_weights(wl)
    x = synth.inputs(wl)
    args = (x["txt"], x["clip"], wl.dims, wl.steps, wl.cfg_scale)
    xc, trace, fresh = O.sample_cfg_cache(x["x0"], x["img_lat"], w, *args, t_cfg=0.5)
    assert fresh == [True, True, False, False]
    assert trace[2][1] is trace[1][1] and trace[3][1] is trace[1][1]
    # the conditional row computed alone is the conditional row of the batch of two
    x_after2 = O.euler_cfg_step(O.euler_cfg_step(x["x0"], *trace[0], wl.cfg_scale, 0.25), *trace[1], wl.cfg_scale, 0.25)
    v_pair = O.dit_forward(np.stack([x_after2, x_after2]), O.build_cond_y(x["img_lat"]), 500.0, w,
                           [O.cross_kv(w, i, *O.context_embed(w, np.stack([x["txt"], 0 * x["txt"]]), x["clip"]))
                            for i in range(wl.dims.blocks)], wl.dims)
    np.testing.assert_allclose(trace[2][0], v_pair[0], atol=1e-12)
    # and it changes the result relative to fresh CFG
    assert np.abs(xc - O.sample(x["x0"], x["img_lat"], w, *args)[0]).max() > 1e-6


def test_cfg_cache_is_exact_at_guidance_scale_one():
    # s = 1: v = v_c whatever v_u is, so caching v_u changes nothing
    wl = synth.TINY_MOE
    w = synth.model_weights(wl)
    x = synth.inputs(wl)
    args = (x["txt"], x["clip"], wl.dims, wl.steps, 1.0)
    xc, _, fresh = O.sample_cfg_cache(x["x0"], x["img_lat"], w, *args, t_cfg=0.6)
    assert fresh == [True, True, False, False]
    np.testing.assert_allclose(xc, O.sample(x["x0"], x["img_lat"], w, *args)[0], atol=1e-12)


# ------------------------------------------------------------------ FP8 building blocks ([WAN] 5.3)
def test_e4m3_round_matches_torch_conversion():
    a = RNG.standard_normal(20000) * np.exp(RNG.uniform(-14, 7, 20000))
    a = a[np.abs(a) <= 448.0]                      # torch's e4m3fn turns overflow into NaN; saturation is pinned below
    # exact ties between neighbouring e4m3 values, both parities
    codes = np.arange(1, 0x7E, dtype=np.uint8)     # positive finite codes below 448
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ties = (vals[:-1] + vals[1:]) / 2
    a = np.concatenate([a, ties, -ties, [0.0, -0.0, 448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10]])
    want = torch.from_numpy(a).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3(a), want)
    # saturation at the largest finite value
    np.testing.assert_array_equal(O.e4m3([464.0, 1e6, -500.0]), [448.0, 448.0, -448.0])


def test_quant_rows_reconstructs_within_half_an_e4m3_step():
    x = (RNG.standard_normal((64, 300)) * np.exp(RNG.uniform(-3, 3, (64, 1)))).astype(np.float32)
    x[5] = 0.0                                      # an all-zero row
    q, s = O.quant_rows_e4m3(x)
    assert s.dtype == np.float32 and s[5] == 1.0 and np.all(q[5] == 0)
    assert np.all(np.abs(q).max(axis=1)[np.arange(64) != 5] == 448.0)   # each row's amax maps to 448
    err = np.abs(q * s[:, None].astype(np.float64) - x)
    # |x/s - q| <= half a step of the e4m3 grid at |x/s| (2^-4 relative, or 2^-10 absolute below 2^-6),
    # plus the fp32 rounding of x / s
    y = np.abs(x / s[:, None])
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(err <= (step / 2 + y * 2.0 ** -23) * s[:, None] + 1e-30)


def test_gemm_fp8_is_the_scaled_integer_dot_product():
    # e4m3 values times 2^9 are integers: the GEMM of the codes is an exact integer product
    qa = O.e4m3(RNG.standard_normal((7, 64)) * 20)
    qb = O.e4m3(RNG.standard_normal((5, 64)) * 20)
    ia, ib = (qa * 512).astype(np.int64), (qb * 512).astype(np.int64)
    assert np.all(ia == qa * 512) and np.all(ib == qb * 512)
    sa, sb, bias = RNG.uniform(0.5, 2, 7), RNG.uniform(0.5, 2, 5), RNG.standard_normal(5)
    want = (ia @ ib.T).astype(np.float64) / 512 ** 2 * sa[:, None] * sb[None, :] + bias
    np.testing.assert_allclose(O.gemm_fp8(qa, sa, qb, sb, bias), want, rtol=1e-15, atol=1e-12)


# ------------------------------------------------------------------ rounding invariants (property-based)
from hypothesis import given, settings, strategies as st  # noqa: E402

_floats = st.floats(min_value=-6e4, max_value=6e4, allow_nan=False, allow_infinity=False, width=64)


@settings(max_examples=300, deadline=None)
@given(st.lists(_floats, min_size=2, max_size=64))
def test_rounding_functions_are_idempotent_monotone_and_odd(xs):
    x = np.sort(np.asarray(xs))
    for fn in (O.bf16, O.fp16, O.e4m3):
        r = fn(x)
        np.testing.assert_array_equal(fn(r), r)                 # values of the format round to themselves
        assert np.all(np.diff(r) >= 0)                          # order is kept
        np.testing.assert_array_equal(fn(-x), -r)               # odd
