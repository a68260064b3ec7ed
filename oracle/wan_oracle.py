"""CPU oracle of the Wan2.1-style I2V DiT denoising step and its CFG Euler sampler.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never calls it and shares no code with it.

Plain, slow and obviously correct: float64 numpy, materialised softmax per
query row, library matmul/erf as the only primitives, no blocking or fusion.
Every function cites the passage of the source pages it follows:

* [I2V]  "图解 Wan2.1 I2V：从一张图到一段视频，模型到底发生了什么" (liyongzhi.xyz)
* [WAN]  "Wan（通义万相）：大规模视频生成基础模型 — 技术深度解析 & Wan2.1 vs Wan2.2对比"
         (devpress.csdn.net)
* [MLQM] "从热词到架构：Wan2.1到底在解决什么问题" (mlqm.cn)

Where the pages are silent the oracle takes the plainest reading; each one is
marked "Reading:" below.  Storage rounding: with ``rnd=True`` the oracle rounds
to bfloat16 (round-to-nearest-even) at exactly the points where the GPU path
stores a bf16 tensor (GEMM operands, q/k/v, attention outputs, FFN hidden),
and to IEEE half where it stores a half tensor (the cross-attention queries
and K/V cache), so a bf16 run is compared with the same function.
Parity pins: see tests/test_oracle_*.py.  Functions whose full output no page
pins ("parity unpinned" against the pages, which print no tensor values):
dit_forward and block_forward.  The tests pin them by invariants (AdaLN-Zero
identity, attention and RoPE special cases), branch by branch, and whole
against a second implementation of the same readings in torch.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

F64 = np.float64


# ---------------------------------------------------------------- storage rounding
def bf16(a) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even (8 significant bits).

    Reading: the pages fix no precision; bf16 storage with round-to-nearest-even
    is the GPU path's storage type.  frexp gives a = m * 2**e with |m| in
    [0.5, 1); keeping 8 significant bits means rounding m * 2**8 to an integer
    (numpy's rint rounds halves to even).
    """
    a = np.asarray(a, dtype=F64)
    m, e = np.frexp(a)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def fp16(a) -> np.ndarray:
    """Round to the nearest IEEE binary16 value, ties to even.

    Normal halves keep 11 significant bits: for a = m * 2**e (|m| in
    [0.5, 1)) the spacing is 2**(e - 11).  Below 2**-14 the spacing stays at
    2**-24 (subnormals).  Results above the largest finite half, 65504, are
    infinite.
    Reading: the pages fix no precision; the bf16 model keeps its
    cross-attention operands (cross queries and the K/V cache) in IEEE half,
    because the text cross-attention softmax is sharp (scores of several
    units) and amplifies the rounding of its operands.
    """
    a = np.asarray(a, dtype=F64)
    _, e = np.frexp(a)
    q = np.maximum(e - 11, -24)
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    return np.where(np.abs(r) > 65504.0, np.copysign(np.inf, a), r)


def _st(a, rnd: bool):
    return bf16(a) if rnd else np.asarray(a, dtype=F64)


def _st16(a, rnd: bool):
    return fp16(a) if rnd else np.asarray(a, dtype=F64)


# ---------------------------------------------------------------- shapes
def token_count(F: int, H: int, W: int) -> int:
    """Tokens of an F-frame H x W video: latent (1+(F-1)/4) x H/8 x W/8, then the
    (1,2,2) patch halves each spatial side ([I2V] 2, 5.1; [WAN] 2.2, 2.5)."""
    T = 1 + (F - 1) // 4
    return T * (H // 16) * (W // 16)


def grid_positions(T: int, Hp: int, Wp: int):
    """Token order l = (f*Hp + y)*Wp + x, the flattening of the Conv3d output grid
    [T, Hp, Wp] ([I2V] 5.1).  Returns the (frame, row, column) of every token."""
    f, y, x = np.meshgrid(np.arange(T), np.arange(Hp), np.arange(Wp), indexing="ij")
    return f.reshape(-1), y.reshape(-1), x.reshape(-1)


# ---------------------------------------------------------------- conditioning y
def mask_frames(T: int, known_pixel_frames=(0,)) -> np.ndarray:
    """Temporal mask m [4, T] of [I2V] 4.1 step 3 (and Q3, Q6).

    A pixel-frame mask of length F = 4(T-1)+1 holds 1 at known frames.  Frame 0
    is repeated 4 times in front of frames 1..F-1, giving 4T entries s, which
    are grouped into consecutive runs of 4: m[c, f] = s[4f + c].
    Reading: the grouping is by consecutive runs (one latent frame = 4 pixel
    frames), which puts all ones of the default mask on latent frame 0.
    """
    F = 4 * (T - 1) + 1
    known = set(int(p) for p in known_pixel_frames)
    pix = np.array([1.0 if p in known else 0.0 for p in range(F)])
    s = np.concatenate([np.repeat(pix[:1], 4), pix[1:]])
    assert s.shape[0] == 4 * T
    m = np.empty((4, T))
    for f in range(T):
        for c in range(4):
            m[c, f] = s[4 * f + c]
    return m


def build_cond_y(img_lat: np.ndarray, known_pixel_frames=(0,)) -> np.ndarray:
    """y = concat(mask [4,T,H,W], image latent [16,T,H,W]) -> [20,T,H,W]
    ([I2V] 4.1 step 4)."""
    C, T, H, W = img_lat.shape
    m = mask_frames(T, known_pixel_frames)
    mask = np.broadcast_to(m[:, :, None, None], (4, T, H, W))
    return np.concatenate([mask, np.asarray(img_lat, F64)], axis=0)


# ---------------------------------------------------------------- elementwise pieces
def silu(x):
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def gelu(x):
    """Exact GELU x * Phi(x) ([I2V] 5.5: Linear -> GELU -> Linear).
    Reading: the erf form (no tanh approximation)."""
    x = np.asarray(x, F64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def linear(x, w, b=None):
    """y = x W^T + b with W stored [out, in]."""
    y = np.asarray(x, F64) @ np.asarray(w, F64).T
    if b is not None:
        y = y + np.asarray(b, F64)
    return y


def layer_norm(x, eps: float, gamma=None, beta=None):
    x = np.asarray(x, F64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, F64)
    if beta is not None:
        y = y + np.asarray(beta, F64)
    return y


def rms_norm(x, eps: float, gamma=None):
    x = np.asarray(x, F64)
    y = x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, F64)
    return y


def adaln_modulate(x, shift, scale, eps: float, norm: str = "layer"):
    """x' = norm(x) * (1 + scale) + shift ([I2V] 5.2).
    Reading: norm is LayerNorm without affine, eps 1e-6 (the page names
    LayerNorm); norm="rms" selects RMSNorm instead."""
    n = layer_norm(x, eps) if norm == "layer" else rms_norm(x, eps)
    return n * (1.0 + np.asarray(scale, F64)) + np.asarray(shift, F64)


# ---------------------------------------------------------------- timestep embedding
def sinusoid(tau: float, dim: int = 256) -> np.ndarray:
    """sinusoidal_embedding_1d(256, t) of [I2V] 5.2.
    Reading: [cos(tau w_i), sin(tau w_i)], w_i = 10000^(-i/128), i = 0..127."""
    half = dim // 2
    w = np.power(10000.0, -np.arange(half, dtype=F64) / half)
    a = float(tau) * w
    return np.concatenate([np.cos(a), np.sin(a)])


def time_mod(wts: dict, tau: float, D: int):
    """Shared time MLP ([I2V] 5.2; [WAN] 2.5 "shared MLP + per-block bias").

    e  = Linear2(SiLU(Linear1(sinusoid(tau))))          [D]
    e0 = time_projection(SiLU(e)) reshaped to [6, D] in the order
         (shift1, scale1, gate1, shift2, scale2, gate2).
    Reading: SiLU activations as in the DiT reference design the page cites.
    """
    es = sinusoid(tau, 256)
    e = linear(silu(linear(es, wts["t1.w"], wts["t1.b"])), wts["t2.w"], wts["t2.b"])
    e0 = linear(silu(e), wts["tp.w"], wts["tp.b"]).reshape(6, D)
    return e, e0


# ---------------------------------------------------------------- 3D RoPE
def rope_split(dh: int):
    """Per-head split of [I2V] 5.3: frame d - 4(d/6), row 2(d/6), column 2(d/6)."""
    s = dh // 6
    return dh - 4 * s, 2 * s, 2 * s


def rope_3d(x, pos_f, pos_y, pos_x):
    """Factorised 3D rotary embedding on x [N, heads, dh] ([I2V] 5.3).

    Each head is cut into segments (frame, row, column) of rope_split(dh)
    channels; each segment gets 1D RoPE with its own coordinate.
    Reading: channel pairs (2j, 2j+1) are (real, imaginary) and pair j of a
    segment of size d_s turns by pos * 10000^(-2j/d_s).
    """
    x = np.asarray(x, F64)
    N, h, dh = x.shape
    out = np.empty_like(x)
    off = 0
    for size, pos in zip(rope_split(dh), (pos_f, pos_y, pos_x)):
        j = np.arange(size // 2, dtype=F64)
        freq = np.power(10000.0, -2.0 * j / size)
        theta = np.asarray(pos, F64)[:, None] * freq[None, :]          # [N, size/2]
        c, s = np.cos(theta)[:, None, :], np.sin(theta)[:, None, :]
        re = x[:, :, off:off + size:2]
        im = x[:, :, off + 1:off + size:2]
        out[:, :, off:off + size:2] = re * c - im * s
        out[:, :, off + 1:off + size:2] = re * s + im * c
        off += size
    return out


# ---------------------------------------------------------------- attention
def attention(q, k, v):
    """softmax(q k^T / sqrt(dh)) v per head, no mask ([I2V] 5.3, 5.4).

    q [Nq, h, dh], k/v [Nk, h, dh] -> [Nq, h, dh].  The softmax is
    materialised per query row (subtracting the row maximum).
    Reading: scale 1/sqrt(dh); no key mask (the pages show none).
    """
    q, k, v = (np.asarray(a, F64) for a in (q, k, v))
    Nq, h, dh = q.shape
    out = np.empty((Nq, h, v.shape[2]))
    for hh in range(h):
        s = (q[:, hh, :] @ k[:, hh, :].T) / math.sqrt(dh)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, hh, :] = p @ v[:, hh, :]
    return out


# ---------------------------------------------------------------- patchify / unpatchify
def patchify(x_in):
    """[B, C, T, H, W] -> [B, L, C*4]: the receptive fields of Conv3d(k=(1,2,2),
    s=(1,2,2)) ([I2V] 5.1), flattened in the weight order (c, kh, kw)."""
    x_in = np.asarray(x_in, F64)
    B, C, T, H, W = x_in.shape
    Hp, Wp = H // 2, W // 2
    p = x_in.reshape(B, C, T, Hp, 2, Wp, 2)
    p = p.transpose(0, 2, 3, 5, 1, 4, 6)              # B, T, Hp, Wp, C, kh, kw
    return p.reshape(B, T * Hp * Wp, C * 4)


def unpatchify(p, T: int, Hp: int, Wp: int, C: int = 16):
    """Inverse of patchify: v[b, c, f, 2y+kh, 2x+kw] = p[b, l, c*4 + kh*2 + kw]
    with l = (f*Hp + y)*Wp + x ([I2V] 5.5 "Head ... and unpatchify").
    Reading: output feature order (c, kh, kw), mirroring the Conv3d weight."""
    p = np.asarray(p, F64)
    B = p.shape[0]
    v = p.reshape(B, T, Hp, Wp, C, 2, 2).transpose(0, 4, 1, 2, 5, 3, 6)
    return v.reshape(B, C, T, 2 * Hp, 2 * Wp)


def patch_embed(x_t, y, w_pe, b_pe, rnd: bool = False):
    """tokens = Conv3d(36, D, (1,2,2), stride (1,2,2))(concat(x_t, y)) as a GEMM
    ([I2V] 4.2 for the 36-channel concat, 5.1 for the patchify).
    x_t [B,16,T,H,W]; y [20,T,H,W] shared by the batch -> [B, L, D].
    y None: the text-to-video model, Conv3d(16, D, ...) of x_t alone ([I2V] 9)."""
    x_t = np.asarray(x_t, F64)
    B = x_t.shape[0]
    if y is None:
        x_in = x_t
    else:
        yb = np.broadcast_to(np.asarray(y, F64)[None], (B,) + np.shape(y))
        x_in = np.concatenate([x_t, yb], axis=1)
    return linear(_st(patchify(x_in), rnd), w_pe, b_pe)


# ---------------------------------------------------------------- context (once per video)
def context_embed(w: dict, txt, clip, rnd: bool = False):
    """Text MLP [n_txt, c_txt] -> [n_txt, D] and CLIP MLPProj [n_img, c_img] ->
    [n_img, D] ([I2V] 7 steps 1-2).  txt is [B, n_txt, c_txt] (the
    unconditional row carries zeroed text, [I2V] Q5); clip is [n_img, c_img],
    or None for the text-to-video model, which has no CLIP branch ([I2V] 9).
    Reading: each MLP is Linear -> GELU -> Linear with biases."""
    t = _st(gelu(linear(txt, w["txt1.w"], w["txt1.b"])), rnd)
    ctx_txt = _st(linear(t, w["txt2.w"], w["txt2.b"]), rnd)
    if clip is None:
        return ctx_txt, None
    i = _st(gelu(linear(clip, w["img1.w"], w["img1.b"])), rnd)
    ctx_img = _st(linear(i, w["img2.w"], w["img2.b"]), rnd)
    return ctx_txt, ctx_img


def cross_kv(w: dict, blk: int, ctx_txt, ctx_img, rnd: bool = False):
    """Per-block cross-attention keys/values of [I2V] 5.4: the text branch uses
    Linear_k / Linear_v, the image branch its own k_img / v_img.  ctx_img None
    (text-to-video, [I2V] 9): text keys and values only."""
    p = f"blk{blk}."
    kv = dict(k_txt=_st16(linear(ctx_txt, w[p + "ck.w"], w[p + "ck.b"]), rnd),
              v_txt=_st16(linear(ctx_txt, w[p + "cv.w"], w[p + "cv.b"]), rnd))
    if ctx_img is not None:
        kv["k_img"] = _st16(linear(ctx_img, w[p + "cki.w"], w[p + "cki.b"]), rnd)
        kv["v_img"] = _st16(linear(ctx_img, w[p + "cvi.w"], w[p + "cvi.b"]), rnd)
    return kv


# ---------------------------------------------------------------- one DiT block
def _mod(e0, w: dict, blk: int):
    """mod = e0 + b_i, rows (shift1, scale1, gate1, shift2, scale2, gate2) ([WAN] 2.5)."""
    return np.asarray(e0, F64) + np.asarray(w[f"blk{blk}.mod"], F64)


def linear_fp8(x, w, b=None):
    """A Linear layer as the FP8 GEMM of [WAN] 5.3: x quantised per row (token),
    W [out, in] per output channel (quant_rows_e4m3), the product of the codes
    exact, both scales applied, then the bias."""
    qx, sx = quant_rows_e4m3(x)
    qw, sw = quant_rows_e4m3(w)
    return gemm_fp8(qx, sx, qw, sw, b)


def _lin(x, w, b, rnd: bool, fp8: bool):
    """The block's Linear layers: on e4m3 operands (fp8), else on operands stored
    as the GPU stores them (rnd) or exact."""
    return linear_fp8(x, w, b) if fp8 else linear(_st(x, rnd), w, b)


def block_qkv(x, e0, w: dict, blk: int, dims, tok, rnd: bool = False, want=("q", "k", "v"), fp8: bool = False):
    """The projections of the self-attention for some tokens of one sample
    ([I2V] 5.2, 5.3 (1) and (2)): x [n, D] are the residual-stream rows of the
    tokens whose sequence indices are `tok` [n];
    h = norm(x)(1 + scale1) + shift1, [q k v] = Linear_qkv(h) (the fused
    projection's rows q; k; v), q and k RMS-normalised over the full width D
    with their gains, split into heads and rotated by the 3D RoPE at each
    token's (frame, row, column) in the grid; v split into heads.
    Returns {name: [n, heads, dh]} for the names in `want`.
    Reading: QK-RMSNorm over D before the head split (the page's
    RMSNorm(Linear_q(x))).  fp8: the projection as an FP8 GEMM whose input h is
    quantised from its fp32 value (not from a bf16 copy)."""
    p = f"blk{blk}."
    D, nh, dh, eps = dims.D, dims.heads, dims.dh, dims.eps
    shift1, scale1 = _mod(e0, w, blk)[:2]
    tok = np.asarray(tok)
    n = len(tok)
    pf, py, px = (a[tok] for a in grid_positions(dims.T, dims.Hp, dims.Wp))
    h = adaln_modulate(x, shift1, scale1, eps, dims.norm)
    wqkv, bqkv = w[p + "qkv.w"], w[p + "qkv.b"]
    out = {}
    for j, name in enumerate(("q", "k", "v")):
        if name not in want:
            continue
        a = _st(_lin(h, wqkv[j * D:(j + 1) * D], bqkv[j * D:(j + 1) * D], rnd, fp8), rnd)
        if name == "v":
            out[name] = a.reshape(n, nh, dh)
        else:
            a = rms_norm(a, eps, w[p + ("gq" if name == "q" else "gk")]).reshape(n, nh, dh)
            out[name] = _st(rope_3d(a, pf, py, px), rnd)
    return out


def block_self_attention(X, e0, w: dict, blk: int, dims, rnd: bool = False, rows=None, fp8: bool = False,
                         attn8: bool = False):
    """The attention output o of a block's self-attention for the token rows
    `rows` of every sample (default all): o = softmax(q k^T / sqrt(dh)) v per
    head over all L keys, heads concatenated -> [B, len(rows), D], the input of
    Linear_o ([I2V] 5.3).  Keys and values cover every token, so the rows are
    exact.  attn8: the FP8 attention (attention_fp8) on the stored q, k, v."""
    X = np.asarray(X, F64)
    B, L, D = X.shape
    rows = np.arange(L) if rows is None else np.asarray(rows)
    o = np.empty((B, len(rows), D))
    for b in range(B):
        kv = block_qkv(X[b], e0, w, blk, dims, np.arange(L), rnd, want=("k", "v"), fp8=fp8)
        q = block_qkv(X[b][rows], e0, w, blk, dims, rows, rnd, want=("q",), fp8=fp8)["q"]
        att = attention_fp8 if attn8 else attention
        o[b] = _st(att(q, kv["k"], kv["v"]).reshape(len(rows), D), rnd)
    return o


def block_after_attention(Xr, o, e0, w: dict, blk: int, kv: dict, dims, rnd: bool = False, fp8: bool = False):
    """The rest of the block for some token rows, given their self-attention
    output o [B, n, D] and their residual-stream rows Xr [B, n, D]
    ([I2V] 5.2-5.5):
    X  += gate1 * Linear_o(o)
    X  += Linear_co(attn(qc, K_img, V_img) + attn(qc, K_txt, V_txt)),
          qc = Linear_cq(LN_affine(X))                (no adaLN, no gate)
    X  += gate2 * Linear_2(GELU(Linear_1(norm(X)(1+scale2)+shift2)))
    Reading: the cross-attention input gets a LayerNorm with affine gains.
    fp8: the four Linear layers as FP8 GEMMs; the norms' outputs are quantised
    from their fp32 values, o, oc and the FFN hidden after their bf16 store.
    fp8 = "no-ffn2": the FFN's second layer stays bf16."""
    p = f"blk{blk}."
    D, nh, dh, eps = dims.D, dims.heads, dims.dh, dims.eps
    Xr = np.asarray(Xr, F64)
    B, n, _ = Xr.shape
    shift1, scale1, gate1, shift2, scale2, gate2 = _mod(e0, w, blk)
    out = np.empty((B, n, D))
    for b in range(B):
        xr = Xr[b] + gate1 * _lin(o[b], w[p + "o.w"], w[p + "o.b"], rnd, fp8)
        # ---- decoupled cross-attention (not modulated, not gated)
        hc = layer_norm(xr, eps, w[p + "cn.g"], w[p + "cn.b"])
        qc = _st16(_lin(hc, w[p + "cq.w"], w[p + "cq.b"], rnd, fp8), rnd).reshape(n, nh, dh)
        kt, vt = kv["k_txt"][b], kv["v_txt"][b]
        o_txt = attention(qc, kt.reshape(-1, nh, dh), vt.reshape(-1, nh, dh))
        if "k_img" in kv:
            ki, vi = kv["k_img"], kv["v_img"]
            o_img = attention(qc, ki.reshape(-1, nh, dh), vi.reshape(-1, nh, dh))
            oc = _st((o_img + o_txt).reshape(n, D), rnd)
        else:   # text-to-video: single-stream cross-attention ([I2V] 9)
            oc = _st(o_txt.reshape(n, D), rnd)
        xr = xr + _lin(oc, w[p + "co.w"], w[p + "co.b"], rnd, fp8)
        # ---- gated FFN
        h2 = adaln_modulate(xr, shift2, scale2, eps, dims.norm)
        u = _st(gelu(_lin(h2, w[p + "f1.w"], w[p + "f1.b"], rnd, fp8)), rnd)
        out[b] = xr + gate2 * _lin(u, w[p + "f2.w"], w[p + "f2.b"], rnd, fp8 and fp8 != "no-ffn2")
    return out


def block_forward(X, e0, w: dict, blk: int, kv: dict, dims, rnd: bool = False, rows=None, fp8: bool = False,
                  attn8: bool = False):
    """One DiT block ([I2V] 5.2-5.5), order self-attention -> cross -> FFN:
    block_self_attention, then block_after_attention.

    X [B, L, D] residual stream; e0 [6, D]; kv from cross_kv (k_txt/v_txt
    [B, n_txt, D], k_img/v_img [n_img, D]).  ``rows`` (optional index array)
    computes the output only for those token rows of every sample; keys and
    values still cover all L tokens, so the result is exact for those rows.
    fp8: the six Linear layers as FP8 GEMMs ([WAN] 5.3), as the GPU's FP8 block.
    attn8: the self-attention as the FP8 attention of [WAN] 5.3.
    """
    X = np.asarray(X, F64)
    rows = np.arange(X.shape[1]) if rows is None else np.asarray(rows)
    o = block_self_attention(X, e0, w, blk, dims, rnd, rows, fp8, attn8)
    return block_after_attention(X[:, rows], o, e0, w, blk, kv, dims, rnd, fp8)


# ---------------------------------------------------------------- head
def head_unpatchify(X, e, w: dict, dims, rnd: bool = False):
    """Head with adaLN and unpatchify ([I2V] 5.5): z = LN(X)(1+sc)+sh with
    (sh, sc) = e + b_head; p = Linear(D -> 16*1*2*2)(z); v = unpatchify(p).
    Reading: shift then scale rows of b_head [2, D], added to e (not e0)."""
    sh = np.asarray(e, F64) + np.asarray(w["head.mod"][0], F64)
    sc = np.asarray(e, F64) + np.asarray(w["head.mod"][1], F64)
    z = _st(adaln_modulate(X, sh, sc, dims.eps, "layer"), rnd)
    p = linear(z, w["head.w"], w["head.b"])
    return unpatchify(p, dims.T, dims.Hp, dims.Wp)


# ---------------------------------------------------------------- whole DiT
def dit_forward(x_t, y, tau: float, w: dict, kvs: list, dims, rnd: bool = False, attn=None, fp8: bool = False,
                attn8: bool = False):
    """v = DiT(concat(x_t, y), tau, context) for a batch ([I2V] 5, 7).
    attn (optional, the attention cache of [WAN] 5.3): a dict with "o", a
    list holding per block the self-attention output o [B, L, D] last
    computed, and "reuse": when true every block takes its stored o instead of
    computing its self-attention; otherwise each block's o is computed and
    stored there."""
    e, e0 = time_mod(w, tau, dims.D)
    X = patch_embed(x_t, y, w["pe.w"], w["pe.b"], rnd)
    for i in range(dims.blocks):
        if attn is None:
            X = block_forward(X, e0, w, i, kvs[i], dims, rnd, fp8=fp8, attn8=attn8)
            continue
        if not attn["reuse"]:
            attn["o"][i] = block_self_attention(X, e0, w, i, dims, rnd)
        X = block_after_attention(X, attn["o"][i], e0, w, i, kvs[i], dims, rnd)
    return head_unpatchify(X, e, w, dims, rnd)


# ---------------------------------------------------------------- flow matching + sampler
def fm_path(x0, x1, t: float):
    """x_t = (1-t) x0 + t x1 with x0 noise and x1 data ([WAN] 2.7)."""
    return (1.0 - t) * np.asarray(x0, F64) + t * np.asarray(x1, F64)


def fm_velocity(x0, x1):
    """v = x1 - x0 ([WAN] 2.7)."""
    return np.asarray(x1, F64) - np.asarray(x0, F64)


def cfg_combine(v_c, v_u, s: float):
    """v = v_u + s (v_c - v_u) ([I2V] 7)."""
    v_c, v_u = np.asarray(v_c, F64), np.asarray(v_u, F64)
    return v_u + s * (v_c - v_u)


def euler_cfg_step(x, v_c, v_u, s: float, dt: float):
    """Explicit Euler step of dx/dt = v from t to t+dt ([WAN] 2.7 "20-50 Euler
    steps"; [MLQM] 3.2), with CFG ([I2V] 7).  v_u None means no guidance."""
    v = np.asarray(v_c, F64) if v_u is None else cfg_combine(v_c, v_u, s)
    return np.asarray(x, F64) + dt * v


def schedule(N: int):
    """Uniform grid t_k = k/N on [0, 1] with dt = 1/N; the model sees
    tau_k = 1000 (1 - t_k).  Reading: the [WAN] 2.7 convention (x0 noise at
    t=0, data at t=1) integrated forward; tau is the noise level x 1000, which
    is the [I2V] 7 schedule (1.0 at noise) on a 0..1000 scale."""
    return [(k / N, 1.0 / N, 1000.0 * (1.0 - k / N)) for k in range(N)]


def sample(x0, img_lat, w: dict, txt, clip, dims, steps: int, cfg_scale: float,
           rnd: bool = False, model=None, known_pixel_frames=(0,)):
    """The inference loop of [I2V] 7: prepare y and the context once, then
    `steps` CFG Euler steps.  The cond row sees the text, the uncond row zeroed
    text with CLIP and y kept ([I2V] Q5).  ``model(x, tau)`` (optional) stands
    in for the DiT and returns (v_c, v_u).  Returns the final latent and the
    per-step velocities.  img_lat and clip None: the text-to-video model
    ([I2V] 9), which has no y and no CLIP context."""
    if model is None:
        y = None if img_lat is None else build_cond_y(img_lat, known_pixel_frames)
        txt2 = np.stack([np.asarray(txt, F64), np.zeros_like(txt, dtype=F64)])
        ctx_txt, ctx_img = context_embed(w, txt2, clip, rnd)
        kvs = [cross_kv(w, i, ctx_txt, ctx_img, rnd) for i in range(dims.blocks)]

        def model(x, tau):
            v = dit_forward(np.stack([x, x]), y, tau, w, kvs, dims, rnd)
            return v[0], v[1]
    x = np.asarray(x0, F64)
    trace = []
    for t, dt, tau in schedule(steps):
        v_c, v_u = model(x, tau)
        trace.append((v_c, v_u))
        x = euler_cfg_step(x, v_c, v_u, cfg_scale, dt)
    return x, trace


def expert_for(noise_level: float, t_moe: float) -> str:
    """Timestep-level MoE of Wan2.2 ([WAN] 7.2): the high-noise expert while the
    noise level exceeds the boundary t_moe, the low-noise expert from there on.
    Reading: the page's t in this passage is the noise level (high noise first,
    in the order of denoising), here 1 - t_k = tau / 1000; its rule for t_moe
    (SNR(t_moe) = SNR_min / 2) is garbled and cannot be evaluated as printed
    (SNR_min is 0 at pure noise), so t_moe is a parameter."""
    return "high" if noise_level > t_moe else "low"


def sample_moe(x0, img_lat, w_high: dict, w_low: dict, txt, clip, dims, steps: int, cfg_scale: float,
               t_moe: float, rnd: bool = False):
    """The sampler of `sample` with two experts of the same architecture
    ([WAN] 7.2): each Euler step evaluates the expert that `expert_for` picks
    for that step's noise level; each expert has its own context projections
    and cross-attention keys and values.  Returns the final latent, the
    per-step velocities and the expert used at each step."""
    y = None if img_lat is None else build_cond_y(img_lat)
    txt2 = np.stack([np.asarray(txt, F64), np.zeros_like(txt, dtype=F64)])
    kvs = {}
    for name, w in (("high", w_high), ("low", w_low)):
        ctx_txt, ctx_img = context_embed(w, txt2, clip, rnd)
        kvs[name] = [cross_kv(w, i, ctx_txt, ctx_img, rnd) for i in range(dims.blocks)]
    ws = {"high": w_high, "low": w_low}
    x = np.asarray(x0, F64)
    trace, used = [], []
    for t, dt, tau in schedule(steps):
        name = expert_for(tau / 1000.0, t_moe)
        v = dit_forward(np.stack([x, x]), y, tau, ws[name], kvs[name], dims, rnd)
        trace.append((v[0], v[1]))
        used.append(name)
        x = euler_cfg_step(x, v[0], v[1], cfg_scale, dt)
    return x, trace, used


def sample_cfg_cache(x0, img_lat, w: dict, txt, clip, dims, steps: int, cfg_scale: float, t_cfg: float,
                     rnd: bool = False):
    """The sampler of `sample` with the CFG cache of [WAN] 5.3 ("skip the
    unconditional path in the late steps").  Reading: while the noise level
    tau / 1000 exceeds t_cfg both rows are evaluated; from the first step at or
    below it only the conditional row is, and the CFG combination reuses the
    last unconditional velocity computed.  Returns the final latent, the
    per-step (v_c, v_u) actually combined, and per step whether v_u was fresh."""
    y = None if img_lat is None else build_cond_y(img_lat)
    txt2 = np.stack([np.asarray(txt, F64), np.zeros_like(txt, dtype=F64)])
    ctx_txt, ctx_img = context_embed(w, txt2, clip, rnd)
    kvs = [cross_kv(w, i, ctx_txt, ctx_img, rnd) for i in range(dims.blocks)]
    kvs_c = [cross_kv(w, i, ctx_txt[:1], ctx_img, rnd) for i in range(dims.blocks)]   # the conditional row alone
    x = np.asarray(x0, F64)
    trace, fresh = [], []
    v_u = None
    for t, dt, tau in schedule(steps):
        if v_u is None or tau / 1000.0 > t_cfg:
            v = dit_forward(np.stack([x, x]), y, tau, w, kvs, dims, rnd)
            v_c, v_u = v[0], v[1]
            fresh.append(True)
        else:
            v_c = dit_forward(x[None], y, tau, w, kvs_c, dims, rnd)[0]
            fresh.append(False)
        trace.append((v_c, v_u))
        x = euler_cfg_step(x, v_c, v_u, cfg_scale, dt)
    return x, trace, fresh


def attn_cache_fresh(k: int, noise_level: float, last_fresh, t_attn: float, interval: int) -> bool:
    """Whether step k recomputes the self-attention under the attention cache
    of [WAN] 5.3 ("reuse attention outputs across steps").  Reading: a step
    recomputes while nothing is stored, while its noise level exceeds t_attn
    (the early steps, where the latent changes fastest), and otherwise once
    `interval` steps have passed since the last recomputation; the steps in
    between reuse.  interval = 1 never reuses."""
    return last_fresh is None or noise_level > t_attn or k - last_fresh >= interval


def sample_attn_cache(x0, img_lat, w: dict, txt, clip, dims, steps: int, cfg_scale: float, t_attn: float,
                      interval: int, rnd: bool = False):
    """The sampler of `sample` with the attention cache of [WAN] 5.3.
    Reading: what is reused is each block's self-attention output o (the
    input of its output projection), per block and per batch row; on a
    reusing step each block skips its norm, q/k/v projection, QK-norm, RoPE
    and self-attention and takes the o stored at the last recomputing step,
    while the gated output projection (with this step's gate), the
    cross-attention and the FFN run as usual.  Returns the final latent, the
    per-step velocities and per step whether it recomputed."""
    y = None if img_lat is None else build_cond_y(img_lat)
    txt2 = np.stack([np.asarray(txt, F64), np.zeros_like(txt, dtype=F64)])
    ctx_txt, ctx_img = context_embed(w, txt2, clip, rnd)
    kvs = [cross_kv(w, i, ctx_txt, ctx_img, rnd) for i in range(dims.blocks)]
    cache = {"o": [None] * dims.blocks, "reuse": False}
    x = np.asarray(x0, F64)
    trace, fresh = [], []
    last = None
    for k, (t, dt, tau) in enumerate(schedule(steps)):
        f = attn_cache_fresh(k, tau / 1000.0, last, t_attn, interval)
        if f:
            last = k
        cache["reuse"] = not f
        v = dit_forward(np.stack([x, x]), y, tau, w, kvs, dims, rnd, attn=cache)
        trace.append((v[0], v[1]))
        fresh.append(f)
        x = euler_cfg_step(x, v[0], v[1], cfg_scale, dt)
    return x, trace, fresh


def sample_diffusion_cache(x0, img_lat, w: dict, txt, clip, dims, steps: int, cfg_scale: float, t_cfg: float,
                           t_attn: float, interval: int, rnd: bool = False):
    """The sampler with both caches of [WAN] 5.3 at once (its "diffusion
    cache"): the CFG cache's rule picks whether a step runs both rows or the
    conditional row alone (reusing the last unconditional velocity); the
    attention cache's rule (one step counter) picks whether the blocks
    recompute their self-attention outputs or reuse them.  Reading: a
    conditional-only step reads and writes the stored outputs of the
    conditional row.  Returns the final latent and per step (both rows?,
    attention recomputed?)."""
    y = None if img_lat is None else build_cond_y(img_lat)
    txt2 = np.stack([np.asarray(txt, F64), np.zeros_like(txt, dtype=F64)])
    ctx_txt, ctx_img = context_embed(w, txt2, clip, rnd)
    kvs = [cross_kv(w, i, ctx_txt, ctx_img, rnd) for i in range(dims.blocks)]
    kvs_c = [cross_kv(w, i, ctx_txt[:1], ctx_img, rnd) for i in range(dims.blocks)]
    o = [None] * dims.blocks              # per block [2, L, D]: row 0 conditional, row 1 unconditional
    x = np.asarray(x0, F64)
    v_u, last, decisions = None, None, []
    for k, (t, dt, tau) in enumerate(schedule(steps)):
        both = v_u is None or tau / 1000.0 > t_cfg
        fresh = attn_cache_fresh(k, tau / 1000.0, last, t_attn, interval)
        if fresh:
            last = k
        if both:
            cache = {"o": o, "reuse": not fresh}
            v = dit_forward(np.stack([x, x]), y, tau, w, kvs, dims, rnd, attn=cache)
            v_c, v_u = v[0], v[1]
        else:
            cache = {"o": [None if a is None else a[:1] for a in o], "reuse": not fresh}
            v_c = dit_forward(x[None], y, tau, w, kvs_c, dims, rnd, attn=cache)[0]
            for i in range(dims.blocks):
                if o[i] is None:
                    o[i] = np.zeros((2,) + cache["o"][i].shape[1:])
                o[i][:1] = cache["o"][i]
        decisions.append((both, fresh))
        x = euler_cfg_step(x, v_c, v_u, cfg_scale, dt)
    return x, decisions


# ---------------------------------------------------------------- FP8 building blocks ([WAN] 5.3)
E4M3_MAX = 448.0


def e4m3(a) -> np.ndarray:
    """Round to the nearest float8 e4m3 value (1 sign, 4 exponent bits with
    bias 7, 3 mantissa bits, no infinities), ties to even, saturating at +-448.
    Normal values keep 4 significant bits: for a = m * 2**e (|m| in [0.5, 1))
    the spacing is 2**(e - 4); below 2**-6 it stays 2**-9 (subnormals)."""
    a = np.asarray(a, dtype=F64)
    _, e = np.frexp(a)
    q = np.maximum(e - 4, -9)
    r = np.ldexp(np.rint(np.ldexp(a, -q)), q)
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def quant_rows_e4m3(x):
    """Per-row (per-token, or per-output-channel for a weight) FP8 quantisation
    of [WAN] 5.3 "FP8 GEMM": scale_r = amax_r / 448 and q = e4m3(x / scale_r), so
    that x ~ scale_r * q.  Reading: the scale and the quotient are computed in
    fp32 (IEEE division, the precision the kernel uses, so both sides take the
    same rounding decisions); an all-zero row gets scale 1.
    Returns (q [rows, K] float64 holding e4m3 values, scale [rows] float32)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x / scale[:, None]).astype(np.float32)
    return e4m3(y), scale


def gemm_fp8(qa, sa, qb, sb, bias=None):
    """C[m, n] = sa[m] * sb[n] * sum_k qa[m, k] qb[n, k] (+ bias[n]): the FP8 GEMM
    with per-row scales of both operands, products and sums in float64."""
    acc = np.asarray(qa, F64) @ np.asarray(qb, F64).T
    out = acc * np.asarray(sa, F64)[:, None] * np.asarray(sb, F64)[None, :]
    return out + np.asarray(bias, F64) if bias is not None else out


# ---------------------------------------------------------------- FP8 attention ([WAN] 5.3)
I8_MAX = 127.0


def quant_rows_int8(x):
    """Per-row symmetric INT8 quantisation for the attention's Q K^T product
    ([WAN] 5.3 "FlashAttention3 FP8": the Q/K inner product in INT8).
    Reading: scale_r = amax_r / 127 and q = round-half-even(x / scale_r), both
    computed in fp32 (IEEE division), as for the e4m3 quantiser; an all-zero row
    gets scale 1.  Returns (codes [rows, K] float64 holding integers in
    [-127, 127], scale [rows] float32)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(I8_MAX), np.float32(1.0)).astype(np.float32)
    y = (x / scale[:, None]).astype(np.float32)
    return np.clip(np.rint(y.astype(F64)), -I8_MAX, I8_MAX), scale


def quant_blocks_int8(x, bk: int = 128):
    """INT8 quantisation with one scale per block of bk consecutive rows (the
    keys of one attention block): each block is quantised as one row by
    quant_rows_int8.  Returns (codes [rows, K], scale [ceil(rows / bk)] float32)."""
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    nb = -(-rows // bk)
    codes, scale = np.empty((rows, K)), np.empty(nb, np.float32)
    for n in range(nb):
        blk = x[n * bk:(n + 1) * bk]
        c, s = quant_rows_int8(blk.reshape(1, -1))
        codes[n * bk:(n + 1) * bk], scale[n] = c.reshape(blk.shape), s[0]
    return codes, scale


def quant_cols_e4m3(x):
    """Per-column (per channel over all rows) e4m3 quantisation of the
    attention's values: quant_rows_e4m3 of the transpose.  Returns (codes
    [rows, K], scale [K] float32)."""
    codes, scale = quant_rows_e4m3(np.asarray(x, dtype=np.float32).T)
    return codes.T, scale


def attention_fp8_head(q, k, v, bk: int = 128, theta: float = 8.0, quant_p: bool = True):
    """One head of the FP8 attention of [WAN] 5.3 ("FlashAttention3 FP8": the
    Q/K inner product in INT8, O = P V in FP8, accumulation across key blocks
    in FP32), q [Nq, dh], k/v [Nk, dh] -> [Nq, dh].

    Reading (the page names the precisions only):
    * Q in INT8 per row (token) and K in INT8 per block of bk keys, so that
      S = (q8 k8^T) sq_r sk_n exactly (integer products); V in e4m3 per channel.
    * The softmax runs blockwise over the keys in order, as the accumulation
      across blocks implies: per block n, logits t = S log2(e) / sqrt(dh)
      (log2 units), the block's row maximum mx; the reference m moves to mx only
      when mx exceeds it by more than theta (log2 units), and then the running
      O and l are scaled by 2^(m_old - m).  p = 2^(t - m) <= 2^theta, its e4m3
      rounding P8 (quant_p) enters O += P8 v8, and the unrounded p enters l.
    * out = O * sv / l.
    With quant_p=False and any theta this is softmax(q k^T / sqrt(dh)) v of the
    dequantised operands exactly; with quant_p the result depends on the
    reference, hence on theta and bk, within e4m3 precision of P."""
    q8, sq = quant_rows_int8(q)
    k8, sk = quant_blocks_int8(k, bk)
    v8, sv = quant_cols_e4m3(v)
    Nq, dh = q8.shape
    c = math.log2(math.e) / math.sqrt(dh)
    m = np.full(Nq, -np.inf)
    l = np.zeros(Nq)
    O = np.zeros((Nq, v8.shape[1]))
    for n in range(len(sk)):
        js = slice(n * bk, min(k8.shape[0], (n + 1) * bk))
        t = (q8 @ k8[js].T) * (np.asarray(sq, F64)[:, None] * F64(sk[n]) * c)
        mx = t.max(axis=1)
        m_new = np.where(mx > m + theta, mx, m)
        alpha = np.exp2(m - m_new)
        p = np.exp2(t - m_new[:, None])
        O = O * alpha[:, None] + (e4m3(p) if quant_p else p) @ v8[js]
        l = l * alpha + p.sum(axis=1)
        m = m_new
    return O * np.asarray(sv, F64)[None, :] / l[:, None]


def attention_fp8(q, k, v, bk: int = 128, theta: float = 8.0, quant_p: bool = True):
    """attention_fp8_head per head: q [Nq, h, dh], k/v [Nk, h, dh] -> [Nq, h, dh].
    The quantisation scales of K and V cover every key of the head, so q may
    hold any subset of the query rows."""
    q, k, v = (np.asarray(a, F64) for a in (q, k, v))
    return np.stack([attention_fp8_head(q[:, hh], k[:, hh], v[:, hh], bk, theta, quant_p)
                     for hh in range(q.shape[1])], axis=1)
