"""Run one libwd kernel at the benchmark's shapes, for timing and profiling.

    python -m flow_matching_video_b200.kernel_cases CASE [--batch B] [--iters N] [--warmup W]

CASE is one of attn_self, attn_cross, attn_fp8 (the FP8 self-attention on
quantised operands), attn_fp8_quantize (the quantisation of q, k, v for it),
gemm_qkv, gemm_o, gemm_ffn1, gemm_ffn2, gemm_ffn1_store (FFN1's shape without the
GELU), euler, euler_hbm, gemm_fp8_qkv,
gemm_fp8_o, gemm_fp8_ffn1, gemm_fp8_ffn2, quant_ffn_hidden, block_480p17 (one
block, 17 frames, L = 7800, batch 1), block_480p81 (one block, L = 32760, batch
2), block_480p81_fp8 (the same block with its six linear layers on e4m3
operands) and block_480p81_fp8attn (and with the FP8 self-attention).
Shapes are those of one block of the 30-block 480p/81-frame model (L = 32760
tokens per sample, D = 1536, 12 heads x 128, FFN 8960, 257 image + 512 text
keys); euler_hbm streams 2^26 elements so that every launch reads HBM.
Inputs are seeded random values; the case prints the mean device time per
launch (CUDA events) and the algorithmic FLOPs or bytes per launch.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from . import build

build.build()
from . import model, synth, wd  # noqa: E402

L, D, H, F, NI, NT = 32760, 1536, 12, 8960, 257, 512

CASES = ("attn_self", "attn_cross", "attn_fp8", "attn_fp8_quantize", "gemm_qkv", "gemm_o", "gemm_ffn1", "gemm_ffn2",
         "gemm_ffn1_store", "euler", "euler_hbm", "gemm_fp8_qkv", "gemm_fp8_o", "gemm_fp8_ffn1", "gemm_fp8_ffn2",
         "quant_ffn_hidden", "block_480p17", "block_480p81", "block_480p81_fp8", "block_480p81_fp8attn")


def bf(*shape):
    return torch.randn(*shape, device="cuda").to(torch.bfloat16)


def hf(*shape):
    return torch.randn(*shape, device="cuda").to(torch.float16)


def make_case(name: str, B: int):
    """(launch, work per launch, "FLOP" or "B", batch the case runs at)."""
    rows = B * L
    if name == "attn_self":
        q, k, v, o = bf(B, L, D), bf(B, L, D), bf(B, L, D), torch.empty(B, L, D, device="cuda", dtype=torch.bfloat16)
        return (lambda: wd.wd_attention(wd.WD_BF16, B, L, H, 128, q, k, v, L, 0, o)), 4.0 * B * L * L * D, "FLOP", B
    if name in ("attn_fp8", "attn_fp8_quantize"):   # q|k|v fused as in the block
        qkv, o = bf(B, L, 3 * D), torch.empty(B, L, D, device="cuda", dtype=torch.bfloat16)
        lay = wd.wd_attention_fp8_layout(B, L, L, H, 128)
        buf = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
        quant = lambda: wd.wd_attention_fp8_quantize(B, L, L, H, 128, qkv, 3 * D, qkv[..., D:], qkv[..., 2 * D:],
                                                     3 * D, buf)
        quant()
        if name == "attn_fp8_quantize":   # bytes: q, k, v read (bf16), q8, k8, v8t written, v read twice
            return quant, B * L * D * (2.0 * 4 + 3.0), "B", B
        return (lambda: wd.wd_attention_fp8(B, L, L, H, 128, buf, o, D)), 4.0 * B * L * L * D, "FLOP", B
    if name == "attn_cross":   # IEEE half operands, bf16 output, as in the block
        q, o = hf(B, L, D), torch.empty(B, L, D, device="cuda", dtype=torch.bfloat16)
        ki, vi, kt, vt = hf(NI, D), hf(NI, D), hf(B, NT, D), hf(B, NT, D)
        return (lambda: wd.wd_attention(wd.WD_F16, B, L, H, 128, q, ki, vi, NI, 1, o, kt, vt, NT, 0),
                4.0 * B * L * (NI + NT) * D, "FLOP", B)
    gemms = {"gemm_qkv": (3 * D, D, wd.EPI_STORE), "gemm_o": (D, D, wd.EPI_RESID),
             "gemm_ffn1": (F, D, wd.EPI_GELU), "gemm_ffn2": (D, F, wd.EPI_RESID),
             "gemm_ffn1_store": (F, D, wd.EPI_STORE)}   # FFN1's shape with a plain bf16 store: the GELU's cost
    if name in gemms:
        N, K, epi = gemms[name]
        A, W, bias = bf(rows, K), bf(N, K) * 0.02, torch.zeros(N, device="cuda")
        out = torch.zeros(rows, N, device="cuda", dtype=torch.float32 if epi == wd.EPI_RESID else torch.bfloat16)
        g = torch.zeros(N, device="cuda")
        return (lambda: wd.wd_gemm(wd.WD_BF16, rows, N, K, A, W, bias, epi, out,
                                   g if epi == wd.EPI_RESID else None)), 2.0 * rows * N * K, "FLOP", B
    fp8 = {"gemm_fp8_qkv": (3 * D, D, wd.EPI_STORE), "gemm_fp8_o": (D, D, wd.EPI_RESID),
           "gemm_fp8_ffn1": (F, D, wd.EPI_GELU), "gemm_fp8_ffn2": (D, F, wd.EPI_RESID)}
    if name in fp8:   # e4m3 operands with per-row scales; FLOPs counted as for the bf16 GEMM
        N, K, epi = fp8[name]
        A, W = bf(rows, K), bf(N, K) * 0.02
        qa, sa = torch.empty((rows, K), dtype=torch.uint8, device="cuda"), torch.empty(rows, device="cuda")
        qw, sw = torch.empty((N, K), dtype=torch.uint8, device="cuda"), torch.empty(N, device="cuda")
        wd.wd_quant_rows_e4m3(wd.WD_BF16, rows, K, A, qa, sa)
        wd.wd_quant_rows_e4m3(wd.WD_BF16, N, K, W, qw, sw)
        bias, g = torch.zeros(N, device="cuda"), torch.zeros(N, device="cuda")
        out = torch.zeros(rows, N, device="cuda", dtype=torch.float32 if epi == wd.EPI_RESID else torch.bfloat16)
        return (lambda: wd.wd_gemm_fp8(rows, N, K, qa, sa, qw, sw, bias, epi, out,
                                       g if epi == wd.EPI_RESID else None)), 2.0 * rows * N * K, "FLOP", B
    if name == "quant_ffn_hidden":   # the FFN hidden activations [B*L, 8960] bf16 -> e4m3 + row scales
        x = bf(rows, F)
        q, sc = torch.empty((rows, F), dtype=torch.uint8, device="cuda"), torch.empty(rows, device="cuda")
        return (lambda: wd.wd_quant_rows_e4m3(wd.WD_BF16, rows, F, x, q, sc)), 3.0 * rows * F + 4.0 * rows, "B", B
    d = synth.Dims(D=D, heads=H, ffn=F, blocks=1, T=21, H=60, W=104, n_txt=NT, c_txt=4096, n_img=NI,
                   c_img=1280, dtype="bf16")
    blocks = {"block_480p17": synth.BLOCK_480P17, "block_480p81": synth.STACK_480P81,
              "block_480p81_fp8": synth.STACK_480P81, "block_480p81_fp8attn": synth.STACK_480P81}
    if name in blocks:   # one DiT block (wd_block_forward) at the workload's batch; FLOPs as in the bench
        wl = blocks[name]
        fp8 = "_fp8" in name   # the block with its linear layers on e4m3 operands
        dd = synth.Dims(**{**wl.dims.__dict__, "blocks": 1})
        net = model.DiT(dd, model.random_weights_on_device(synth.Workload(wl.name, dd, wl.batch, wl.seed), "cuda"),
                        wl.batch, fp8=fp8, fp8_attention=name.endswith("attn"))
        x = synth.inputs(wl)
        txt = torch.from_numpy(np.stack([x["txt"], 0 * x["txt"]][:wl.batch])).to("cuda", torch.bfloat16)
        net.prepare_context(txt, torch.from_numpy(x["clip"]).to("cuda", torch.bfloat16))
        net.X.normal_()
        net.e0.normal_(std=0.1)
        Lb, Db, Fb = dd.L, dd.D, dd.ffn
        flops = wl.batch * (2.0 * Lb * Db * (6 * Db + 2 * Fb) + 4.0 * Lb * Lb * Db + 4.0 * Lb * (dd.n_img + dd.n_txt) * Db)
        if fp8:
            return (lambda: wd.wd_block_forward_fp8(net.cd, net.block_w[0], net.block_w8[0], net.e0, net.kv[0],
                                                    wl.batch, net.X, net.ws)), flops, "FLOP", wl.batch
        return (lambda: wd.wd_block_forward(net.cd, net.block_w[0], net.e0, net.kv[0], wl.batch, net.X, net.ws)), \
            flops, "FLOP", wl.batch
    if name in ("euler", "euler_hbm"):
        # euler: the step's latent (33.5 MB, L2-resident between launches);
        # euler_hbm: 2^26 elements (1.07 GB of traffic), so every launch streams HBM
        n = 16 * 21 * 60 * 104 if name == "euler" else 1 << 26
        x, vc, vu = (torch.randn(n, device="cuda") for _ in range(3))
        return (lambda: wd.wd_euler_cfg_step(x, vc, vu, 5.0, 1 / 12)), 16.0 * n, "B", B
    raise SystemExit(f"unknown case {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=CASES)
    ap.add_argument("--batch", type=int, default=2)
    ap.add_argument("--iters", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    a = ap.parse_args()
    torch.manual_seed(0)
    run, work, unit, batch = make_case(a.case, a.batch)
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(a.iters):
        run()
    e.record()
    torch.cuda.synchronize()
    wd.wd_check()
    ms = s.elapsed_time(e) / a.iters
    rate = work / (ms / 1e3) / (1e12 if unit == "FLOP" else 1e9)
    print(f"{a.case} batch={batch}: {ms:.4f} ms/launch, {work:.4g} {unit}/launch, "
          f"{rate:.1f} {'TFLOP/s' if unit == 'FLOP' else 'GB/s'}")


if __name__ == "__main__":
    main()
