"""Seeded synthetic inputs and random-init weights for the Wan2.1-style I2V DiT.

This module holds shapes and random numbers only: no step of the method's
arithmetic lives here.  Both the CPU oracle (through the tests) and the CUDA
path draw their inputs from it, so the two sides see identical values.

Streams: every tensor is drawn from its own PCG64 stream keyed by
(seed, crc32(name)), so adding a tensor never shifts another one.

Shapes follow the I2V pipeline of "图解 Wan2.1 I2V" (liyongzhi.xyz):
text tokens [512, 4096] (section 3.1), CLIP tokens [257, 1280] (section 3.2),
latent [16, T, H/8, W/8] (section 2), 36-channel DiT input (section 4.2).
Weights are N(0, 0.02); norm gains are 1 + N(0, 0.02) so that the QK-norms do
not collapse q and k to zero (a literal N(0, 0.02) gain would make attention
uniform and hide indexing mistakes).
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, replace

import numpy as np

LATENT_C = 16          # VAE latent channels
MASK_C = 4             # mask channels (VAE temporal stride)
IN_C = LATENT_C + MASK_C + LATENT_C   # 36-channel DiT input
PATCH_K = IN_C * 1 * 2 * 2            # 144 values per (1,2,2) patch
PATCH_K_T2V = LATENT_C * 1 * 2 * 2    # 64: the text-to-video model embeds x_t alone
OUT_P = LATENT_C * 1 * 2 * 2          # 64 head outputs per token
T_EMB = 256            # sinusoidal timestep embedding width
WEIGHT_STD = 0.02


@dataclass(frozen=True)
class Dims:
    D: int
    heads: int
    ffn: int
    blocks: int
    T: int          # latent frames
    H: int          # latent height
    W: int          # latent width
    n_txt: int
    c_txt: int
    n_img: int
    c_img: int
    dtype: str      # "f32" or "bf16": matrix / activation storage type
    norm: str = "layer"   # adaLN norm: "layer" (default) or "rms"
    eps: float = 1e-6

    @property
    def dh(self) -> int:
        return self.D // self.heads

    @property
    def Hp(self) -> int:
        return self.H // 2

    @property
    def Wp(self) -> int:
        return self.W // 2

    @property
    def L(self) -> int:
        return self.T * self.Hp * self.Wp

    @property
    def t2v(self) -> bool:
        """Text-to-video model ("图解 Wan2.1 I2V" section 9): no image branch."""
        return self.n_img == 0

    @property
    def patch_k(self) -> int:
        return PATCH_K_T2V if self.t2v else PATCH_K

    @property
    def F_pix(self) -> int:
        """Pixel frames that a latent of T frames encodes: T = 1 + (F-1)/4."""
        return 4 * (self.T - 1) + 1


@dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    batch: int          # 1, or 2 for a cond/uncond pair
    seed: int
    steps: int = 1      # Euler steps of the sampler
    cfg_scale: float = 5.0
    txt_valid: tuple = (512, 512)   # text rows >= n_valid are zero; n_valid ~ U[lo, hi]
    t_moe: float = None   # two experts (timestep MoE): the high-noise one while the noise level exceeds t_moe


# The five workloads: a tiny fp32 model, one bf16 block at 480p/17 frames,
# the 30-block bf16 stack at 480p/81 frames, the wide 40-block stack at
# 720p/81 frames, and the 12-step sampling loop of the 30-block model.
TINY = Workload("tiny-fp32-2blk-L32",
                Dims(D=128, heads=4, ffn=512, blocks=2, T=2, H=8, W=8,
                     n_txt=16, c_txt=64, n_img=9, c_img=32, dtype="f32"),
                batch=2, seed=1001, steps=2, cfg_scale=5.0, txt_valid=(16, 16))
BLOCK_480P17 = Workload("bf16-1blk-D1536-L7800",
                        Dims(D=1536, heads=12, ffn=8960, blocks=1, T=5, H=60, W=104,
                             n_txt=512, c_txt=4096, n_img=257, c_img=1280, dtype="bf16"),
                        batch=1, seed=1002, txt_valid=(16, 512))
STACK_480P81 = Workload("bf16-30blk-D1536-L32760-cfg",
                        Dims(D=1536, heads=12, ffn=8960, blocks=30, T=21, H=60, W=104,
                             n_txt=512, c_txt=4096, n_img=257, c_img=1280, dtype="bf16"),
                        batch=2, seed=1003, steps=1, cfg_scale=5.0)
WIDE_720P81 = Workload("bf16-40blk-D5120-L75600-cfg",
                       Dims(D=5120, heads=40, ffn=13824, blocks=40, T=21, H=90, W=160,
                            n_txt=512, c_txt=4096, n_img=257, c_img=1280, dtype="bf16"),
                       batch=2, seed=1004, steps=1, cfg_scale=5.0)
SAMPLE_480P81 = replace(STACK_480P81, name="bf16-30blk-L32760-12step-cfg", seed=1005, steps=12)
# A small bf16 model with 128-wide heads (so every tensor-core kernel runs) and
# a ragged token grid (L = 3*5*7 = 105): smoke runs and fast parity checks.
SMALL_BF16 = Workload("small-bf16-dh128-L105",
                      Dims(D=256, heads=2, ffn=512, blocks=2, T=3, H=10, W=14, n_txt=24, c_txt=64,
                           n_img=9, c_img=32, dtype="bf16"),
                      batch=2, seed=1012, steps=1, txt_valid=(5, 24))

# Text-to-video counterparts ("图解 Wan2.1 I2V" section 9: 16 input channels, text-only
# cross-attention, no CLIP branch), and the two-expert timestep MoE sampler of
# Wan2.2 ("Wan（通义万相）..." 7.2) on the tiny model.
TINY_T2V = replace(TINY, name="tiny-fp32-2blk-L32-t2v", dims=replace(TINY.dims, n_img=0, c_img=0), seed=1021)
SMALL_BF16_T2V = replace(SMALL_BF16, name="small-bf16-dh128-L105-t2v", dims=replace(SMALL_BF16.dims, n_img=0, c_img=0),
                         seed=1022)
STACK_480P81_T2V = replace(STACK_480P81, name="bf16-30blk-D1536-L32760-t2v-cfg",
                           dims=replace(STACK_480P81.dims, n_img=0, c_img=0), seed=1023)
TINY_MOE = replace(TINY, name="tiny-fp32-2blk-L32-moe", seed=1031, steps=4, t_moe=0.6)

WORKLOADS = {w.name: w for w in (TINY, BLOCK_480P17, STACK_480P81, WIDE_720P81, SAMPLE_480P81, SMALL_BF16,
                                 TINY_T2V, SMALL_BF16_T2V, STACK_480P81_T2V, TINY_MOE)}


def experts(wl: Workload):
    """(high-noise, low-noise) expert workloads of a timestep-MoE sampler: the
    same shapes and inputs, weights from separate seeds."""
    return replace(wl, seed=wl.seed), replace(wl, seed=wl.seed + 500)


def stream(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(name.encode())])))


def _to_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    """float32 array holding values exactly representable in the storage type."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "bf16":
        import torch
        a = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    return a


def normal(seed: int, name: str, shape, std: float = 1.0, mean: float = 0.0,
           dtype: str = "f32") -> np.ndarray:
    a = stream(seed, name).standard_normal(size=shape) * std + mean
    return _to_storage(a, dtype)


def model_weights(wl: Workload, blocks=None) -> dict:
    """Random-init weights for every tensor of the DiT (host, float32 arrays).

    Matrices are [out, in] (Linear convention) and hold values representable in
    dims.dtype; biases, gains and modulation biases are plain float32.
    ``blocks`` limits which block indices are generated (default: all).
    """
    d, s = wl.dims, wl.seed
    D, F, dt = d.D, d.ffn, d.dtype
    std = WEIGHT_STD
    w = {}
    # shared time MLP and projection (always float32)
    w["t1.w"] = normal(s, "t1.w", (D, T_EMB), std)
    w["t1.b"] = normal(s, "t1.b", (D,), std)
    w["t2.w"] = normal(s, "t2.w", (D, D), std)
    w["t2.b"] = normal(s, "t2.b", (D,), std)
    w["tp.w"] = normal(s, "tp.w", (6 * D, D), std)
    w["tp.b"] = normal(s, "tp.b", (6 * D,), std)
    # patch embedding Conv3d(36, D, (1,2,2)) flattened to [D, 36*1*2*2]
    w["pe.w"] = normal(s, "pe.w", (D, d.patch_k), std, dtype=dt)
    w["pe.b"] = normal(s, "pe.b", (D,), std)
    # text and CLIP projections (the text-to-video model has no CLIP branch)
    w["txt1.w"] = normal(s, "txt1.w", (D, d.c_txt), std, dtype=dt)
    w["txt1.b"] = normal(s, "txt1.b", (D,), std)
    w["txt2.w"] = normal(s, "txt2.w", (D, D), std, dtype=dt)
    w["txt2.b"] = normal(s, "txt2.b", (D,), std)
    if not d.t2v:
        w["img1.w"] = normal(s, "img1.w", (D, d.c_img), std, dtype=dt)
        w["img1.b"] = normal(s, "img1.b", (D,), std)
        w["img2.w"] = normal(s, "img2.w", (D, D), std, dtype=dt)
        w["img2.b"] = normal(s, "img2.b", (D,), std)
    mats = (("qkv", (3 * D, D)), ("o", (D, D)), ("cq", (D, D)), ("ck", (D, D)), ("cv", (D, D)),
            ("cki", (D, D)), ("cvi", (D, D)), ("co", (D, D)), ("f1", (F, D)), ("f2", (D, F)))
    for i in (range(d.blocks) if blocks is None else blocks):
        p = f"blk{i}."
        for nm, shp in mats:
            if d.t2v and nm in ("cki", "cvi"):
                continue
            w[p + nm + ".w"] = normal(s, p + nm + ".w", shp, std, dtype=dt)
            w[p + nm + ".b"] = normal(s, p + nm + ".b", (shp[0],), std)
        w[p + "gq"] = normal(s, p + "gq", (D,), std, mean=1.0)
        w[p + "gk"] = normal(s, p + "gk", (D,), std, mean=1.0)
        w[p + "cn.g"] = normal(s, p + "cn.g", (D,), std, mean=1.0)
        w[p + "cn.b"] = normal(s, p + "cn.b", (D,), std)
        w[p + "mod"] = normal(s, p + "mod", (6, D), std)
    w["head.mod"] = normal(s, "head.mod", (2, D), std)
    w["head.w"] = normal(s, "head.w", (OUT_P, D), std, dtype=dt)
    w["head.b"] = normal(s, "head.b", (OUT_P,), std)
    return w


def inputs(wl: Workload) -> dict:
    """Seeded per-video inputs: x0 noise, image latent, text and CLIP tokens."""
    d, s = wl.dims, wl.seed
    x = {}
    x["x0"] = normal(s, "x0", (LATENT_C, d.T, d.H, d.W))
    x["img_lat"] = normal(s, "img_lat", (LATENT_C, d.T, d.H, d.W))
    txt = normal(s, "txt", (d.n_txt, d.c_txt), dtype=d.dtype)
    lo, hi = wl.txt_valid
    n_valid = int(stream(s, "txt_valid").integers(lo, hi + 1)) if hi > lo else min(hi, d.n_txt)
    txt[n_valid:] = 0.0
    x["txt"] = txt
    x["txt_valid"] = n_valid
    if not d.t2v:
        x["clip"] = normal(s, "clip", (d.n_img, d.c_img), dtype=d.dtype)
    return x


def device_normal(shape, std, mean, seed, name, device, torch_dtype):
    """Seeded N(mean, std) tensor drawn directly on a device (large benchmark weights)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((seed << 32) ^ zlib.crc32(name.encode()))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std).add_(mean)
    return t.to(torch_dtype)
