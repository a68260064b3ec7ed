#!/usr/bin/env python
"""Benchmark of the I2V DiT denoising step on B200.

One step = one CFG Euler step of the 30-block bf16 DiT (D=1536, 12 heads x
128, FFN 8960) on an 81-frame 480x832 video: latent [16, 21, 60, 104],
L = 32760 tokens, batch 2 (text-conditioned and zeroed-text rows), i.e. the
time MLP, patch embedding, 30 blocks, head/unpatchify and the CFG Euler
update, all in libwd's kernels.  Inputs and weights are seeded synthetic
values of the real shapes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torch.distributed.run: every rank runs its own video
(independent problems, no collective on the data path: weak scaling).
Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle (the
reference arm of this method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from dataclasses import replace

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DiT block tokens/s & TFLOP/s (% BF16 peak) at L=32760; s per CFG Euler step"
DEFAULT_WORKLOAD = "bf16-30blk-D1536-L32760-cfg"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def block_flops(d) -> dict:
    """Algorithmic FLOPs of one block for one sample: 2MNK per GEMM, 4 L^2 D for
    the self-attention, 4 L (n_img + n_txt) D for the cross-attention."""
    L, D, F = d.L, d.D, d.ffn
    return {"gemm": 2.0 * L * D * (6 * D + 2 * F), "attn_self": 4.0 * L * L * D,
            "attn_cross": 4.0 * L * (d.n_img + d.n_txt) * D}


def step_flops(d, batch) -> float:
    f = block_flops(d)
    extra = 2.0 * d.L * d.patch_k * d.D + 2.0 * d.L * d.D * 64      # patch embedding + head
    return batch * (d.blocks * sum(f.values()) + extra)


# ---------------------------------------------------------------------- clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id=None):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------- CPU oracle rate
class OracleSample:
    """A bounded sample of the workload for timing the CPU oracle: one sample
    (batch row), one block, at the full token count L."""

    def __init__(self, wl):
        import numpy as np
        from oracle import wan_oracle as O
        from flow_matching_video_b200 import synth
        self.O, self.np = O, np
        self.d1 = replace(wl.dims, blocks=1)
        self.w = synth.model_weights(wl, blocks=[0])
        x = synth.inputs(wl)
        y = None if wl.dims.t2v else O.build_cond_y(x["img_lat"])
        self.X = O.patch_embed(x["x0"][None], y, self.w["pe.w"], self.w["pe.b"], rnd=True)
        _, self.e0 = O.time_mod(self.w, 1000.0, self.d1.D)
        ctx_t, ctx_i = O.context_embed(self.w, x["txt"][None], None if wl.dims.t2v else x["clip"], rnd=True)
        self.kv = O.cross_kv(self.w, 0, ctx_t, ctx_i, rnd=True)
        # first call pays allocation and BLAS start-up; not part of any rate
        self.block(self.np.arange(8))

    def block(self, rows):
        return self.O.block_forward(self.X, self.e0, self.w, 0, self.kv, self.d1, rnd=True, rows=rows)

    def rate(self, rows_a=64, rows_b=576, seed=0):
        """The block is computed exactly for rows_a, then rows_b token rows (keys
        and values always cover all L tokens).  The two times give the work
        shared by all rows (the K/V projections) and the per-row work; a full
        block costs shared + L * per_row.  Returns (tokens/s, details)."""
        rng = self.np.random.default_rng(seed)
        L = self.d1.L
        times = []
        for n in (rows_a, rows_b):
            rows = self.np.sort(rng.choice(L, n, replace=False))
            t0 = time.perf_counter()
            self.block(rows)
            times.append(time.perf_counter() - t0)
        per_row = max((times[1] - times[0]) / (rows_b - rows_a), 0.0)
        shared = max(times[0] - rows_a * per_row, 0.0)
        t_block = shared + L * per_row
        return L / t_block, {"t_rows_a": times[0], "t_rows_b": times[1], "shared_s": shared,
                             "per_row_s": per_row, "t_block_est_s": t_block}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ---------------------------------------------------------------------- multi-rank reduction
def reduce_over_ranks(ms_local: float, tokens_local: float, world: int, device=None):
    """Step time = max over ranks; throughput = all ranks' tokens / that time.
    Every rank takes the same collective calls (one all_reduce MAX, one SUM)."""
    import torch
    ms, tokens = ms_local, tokens_local
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms_local], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        n = torch.tensor([tokens_local], dtype=torch.float64, device=device)
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
        tokens = float(n.item())
    return ms, tokens / (ms / 1e3)


# ---------------------------------------------------------------------- reference arm
def run_reference(args, rank):
    if rank != 0:
        return 0
    from flow_matching_video_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    rates, walls, details = [], [], None
    sample = OracleSample(wl)
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r, det = sample.rate(seed=i)
        if i >= args.warmup:
            rates.append(r)
            walls.append(time.perf_counter() - t0)
            details = det
    value = statistics.mean(rates)
    d = wl.dims
    s_step = wl.batch * d.blocks * d.L / value   # a whole CFG step at that rate (not run)
    sample = (f"one sample, one block at L={d.L}: 64 and 576 token rows computed exactly in fp64 (K/V over "
              f"all tokens); full-block time extrapolated as shared + L * per-row")
    # ms_per_step: the wall time of one step as run (one bounded sample); value: the full block's
    # extrapolated block-tokens/s, the workload's throughput
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(walls),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens": d.L, "batch": wl.batch, "blocks": d.blocks},
            "step_is": "one bounded sample (see cpu_baseline.sample); value is extrapolated to the full block",
            "s_per_cfg_step_extrapolated": s_step,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample, "detail": details},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------- our arm
def traffic_for(kernel: str, src_path: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source
    is unchanged since the capture (profiles/traffic.json records its hash)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec:
        return None
    h = hashlib.sha256(open(src_path, "rb").read()).hexdigest()[:16]
    return rec.get("bytes_per_launch") if rec.get("source_sha") == h else None


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from flow_matching_video_b200 import build, synth
    build.build()
    from flow_matching_video_b200 import model, wd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = synth.WORKLOADS[args.workload]
    d = wl.dims
    B = wl.batch
    mode = "cfg-split" if args.cfg_split else ("ulysses" if args.seq_parallel else "replicas")
    if mode == "cfg-split" and world != 2:
        raise SystemExit("--cfg-split runs one video's two CFG rows on exactly two GPUs (--gpus 2)")
    torch.manual_seed(0)
    weights = model.random_weights_on_device(wl, dev)
    # replicas: an independent video per rank; the split modes: one video shared by all ranks
    x = synth.inputs(replace(wl, seed=wl.seed + 7919 * rank) if mode == "replicas" else wl)
    tdt = torch.bfloat16 if d.dtype == "bf16" else torch.float32
    txt = torch.from_numpy(np.stack([x["txt"], np.zeros_like(x["txt"])])).to(dev, tdt)
    clip = None if d.t2v else torch.from_numpy(x["clip"]).to(dev, tdt)
    attn_cache = None
    if mode == "cfg-split":
        # rank 0 evaluates the text row, rank 1 the zeroed-text row, each with a batch-1 model
        from flow_matching_video_b200.cfg_split import CfgSplit
        net = model.DiT(d, weights, 1, dev)
        net.prepare_context(txt[rank:rank + 1].contiguous(), clip)
        runner = CfgSplit(net)
        rows_local = 1
    elif mode == "ulysses":
        from flow_matching_video_b200.seq_parallel import SeqParallelDiT
        net = model.DiT(d, weights, B, dev)
        net.prepare_context(txt, clip)
        runner = SeqParallelDiT(net, rank, world, ring=args.ring)
        rows_local = B / world       # each rank carries 1/world of the tokens through the blocks
    else:
        if args.cfg_cache is not None and args.attn_cache is not None:   # both caches ("diffusion cache")
            t_attn, interval = args.attn_cache
            runner = model.DiffusionCache(d, weights, args.cfg_cache, t_attn, int(interval), dev)
            net, attn_cache = runner.cfg.pair, runner.attn
        elif args.cfg_cache is not None:   # the sampler with the CFG cache: late steps run the conditional row alone
            runner = model.CfgCache(d, weights, args.cfg_cache, dev)
            net = runner.pair
        elif args.attn_cache is not None:   # the sampler with the attention cache
            t_attn, interval = args.attn_cache
            runner = attn_cache = model.AttnCache(d, weights, t_attn, int(interval), B, dev)
            net = runner.net
        else:
            runner = net = model.DiT(d, weights, B, dev, fp8=args.fp8 is not None,
                                     fp8_ffn2=not (args.fp8 or "").startswith("no-ffn2"),
                                     fp8_attention=(args.fp8 or "").endswith("+attn"))
        runner.prepare_context(txt, clip)
        rows_local = B
    y = None if d.t2v else net.build_cond_y(torch.from_numpy(x["img_lat"]).to(dev))
    x_host = torch.from_numpy(x["x0"]).pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()
    n_rows = 1 if mode == "cfg-split" else 2
    xb = torch.empty((n_rows,) + tuple(x_host.shape), device=dev)
    xb.copy_(x_host.expand_as(xb))
    n_sched = 12
    sched = [(k / n_sched, 1.0 / n_sched, 1000.0 * (1 - k / n_sched)) for k in range(n_sched)]
    stream = torch.cuda.current_stream(dev)
    fresh_steps = []   # attention cache: whether each timed step recomputed the attention

    def step(i):
        _, dt, tau = sched[i % n_sched]
        if attn_cache is not None:
            fresh_steps.append(attn_cache.fresh(tau))
        if mode == "cfg-split":
            runner.cfg_euler_step(xb[0], y, tau, dt, wl.cfg_scale)
        else:
            runner.cfg_euler_step(xb, y, tau, dt, wl.cfg_scale)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    wd.wd_check()
    torch.cuda.synchronize()
    barrier()

    # ------------------------------------------------ device-timed region
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = Clocks(gpu_id)
    clocks.start()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    wd.wd_check()
    tokens_step = rows_local * d.L * d.blocks
    ms, value = reduce_over_ranks(e0.elapsed_time(e1) / args.steps, tokens_step, world, dev)
    timed_fresh = list(fresh_steps[args.warmup:args.warmup + args.steps])

    # ------------------------------------------------ the same steps again with per-launch events
    # (kernel shares, launch count and the live roofline; kept out of the timed region above)
    wd.wd_trace_read()
    wd.wd_trace_enable(True)
    torch.cuda.synchronize()
    barrier()
    for i in range(args.steps):
        step(args.warmup + i)
    torch.cuda.synchronize()
    barrier()
    wd.wd_trace_enable(False)
    tr = wd.wd_trace_read()
    wd.wd_check()

    # ------------------------------------------------ end to end through the API, host buffers
    torch.cuda.synchronize()
    barrier()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for i in range(args.steps):
        xb[0].copy_(x_host, non_blocking=True)
        if n_rows == 2:
            xb[1].copy_(xb[0])
        step(i)
        out_host.copy_(xb[0], non_blocking=True)
    h1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e, value_e2e = reduce_over_ranks(h0.elapsed_time(h1) / args.steps, tokens_step, world, dev)
    if not np.all(np.isfinite(out_host.numpy())):
        raise RuntimeError("non-finite latent after the timed steps")

    if rank != 0:
        return 0
    pk = peaks()
    wbytes = sum(t.numel() * t.element_size() for t in weights.values())
    # the whole job's algorithmic work per step: one CFG step (both rows) per video
    flops = step_flops(d, B) * (world if mode == "replicas" else 1)
    cache_note = None
    if args.cfg_cache is not None or attn_cache is not None:
        # the work each timed step did: a step of the CFG cache that ran the conditional row alone
        # does half of a CFG step; a step of the attention cache that reused the attention outputs
        # skips, per block and row, the q/k/v projection and the self-attention
        per_row = step_flops(d, B) / B
        skipped_row = d.blocks * (2.0 * d.L * d.D * 3 * d.D + block_flops(d)["attn_self"])
        work, n_both = 0.0, 0
        for i in range(args.steps):
            both = args.cfg_cache is None or sched[(args.warmup + i) % n_sched][2] / 1000.0 > args.cfg_cache
            rows = B if both else 1
            n_both += both
            reuse = attn_cache is not None and not timed_fresh[i]
            work += rows * (per_row - (skipped_row if reuse else 0.0))
        flops = work / args.steps * (world if mode == "replicas" else 1)
        cache_note = {}
        if args.cfg_cache is not None:
            cache_note.update(t_cfg=args.cfg_cache, steps_with_both_rows=n_both,
                              steps_conditional_only=args.steps - n_both)
        if attn_cache is not None:
            reuse = sum(1 for f in timed_fresh if not f)
            cache_note.update(t_attn=attn_cache.t_attn, interval=attn_cache.interval,
                              steps_recomputing=len(timed_fresh) - reuse, steps_reusing=reuse)
    tflops = flops / (ms / 1e3) / 1e12
    # roofline of the dominant kernel (self-attention), timed live with events
    n_att, ms_att = tr["attn_self"]
    avg_att = ms_att / max(n_att, 1)
    att_flops = (1 if mode == "cfg-split" else B) * block_flops(d)["attn_self"] / (world if mode == "ulysses" else 1)
    achieved = att_flops / (avg_att / 1e3) / 1e12
    peak_s = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    # the FP8 attention's products run at twice the bf16 rate (the nominal int8 / e4m3 : bf16 ratio)
    attn8 = (args.fp8 or "").endswith("+attn")
    peak_att = 2 * peak_s if attn8 else peak_s
    share = {k: round(v[1] / max(sum(u[1] for u in tr.values()), 1e-9), 4) for k, v in tr.items()}
    # the event-timed kernels of one step (traced re-run); ms_per_step minus this is time between kernels
    kernel_ms = sum(v[1] for v in tr.values()) / args.steps
    launches = sum(v[0] for v in tr.values())
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, det = OracleSample(wl).rate()
        cpu = {"value": rate, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"one sample, one block at L={d.L}: 64 and 576 token rows computed exactly in fp64 "
                          f"(K/V over all tokens); full block extrapolated as shared + L * per-row"),
               "detail": det}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak" if mode == "replicas" else "strong",
        "vs_baseline": None, "dtype": fp8_label(args.fp8), "data": "synthetic",
        "config": {"workload": wl.name, "video": f"{4 * (d.T - 1) + 1} frames {8 * d.H}x{8 * d.W}",
                   "latent": [16, d.T, d.H, d.W],
                   "tokens": d.L, "batch": B, "blocks": d.blocks, "D": d.D, "heads": d.heads, "ffn": d.ffn,
                   "parallelism": ("single GPU" if world == 1 and mode == "replicas" else
                                   {"replicas": f"replicas x{world}", "cfg-split": "CFG rows split over 2 GPUs",
                                    "ulysses": (f"Ulysses sequence parallel x{world}" if args.ring == 1 else
                                                f"Ulysses x{world // args.ring} inside {args.ring} ring groups")}[mode]),
                   "l2": (f"no flush: per-step working set ({wbytes / 1e9:.1f} GB weights, "
                          f"{net.X.numel() * 4 / 1e9:.1f} GB residual stream) exceeds L2")},
        "tflops": tflops, "pct_bf16_peak": tflops / pk["bf16_tflops"],
        "pct_bf16_peak_sustained": tflops / peak_s, "s_per_step": ms / 1e3,
        "s_per_video_latent": ms / 1e3 * wl.steps,   # the workload's Euler steps of one video
        "e2e": {"value": value_e2e, "unit": "tokens/s",
                "h2d_bytes_per_step": x_host.numel() * 4, "d2h_bytes_per_step": out_host.numel() * 4},
        "gpu_launches": launches,
        "roofline": {"bound": "tensor",
                     "kernel": ("attention_fp8 self (k_attn_f8: INT8 Q K^T, e4m3 P V)" if attn8 else
                                "attention_tc self (k_attn_tc<2,1,bf16>)"),
                     "achieved": achieved, "peak": peak_att, "unit": "TFLOP/s", "frac": achieved / peak_att,
                     "peak_source": (f"{pk['_source']} bf16 sustained x 2 (nominal int8/e4m3 : bf16 ratio)" if attn8
                                     else f"{pk['_source']} bf16 sustained"),
                     "flops_per_launch": att_flops, "avg_launch_ms": avg_att, "launches": n_att,
                     "traffic": (traffic_for("attn_self_f8", os.path.join(ROOT, "flow_matching_video_b200", "csrc",
                                                                          "k_attn_f8.cu")) if attn8 else
                                 traffic_for("attn_self", os.path.join(ROOT, "flow_matching_video_b200", "csrc",
                                                                       "k_attn_tc.cu")))},
        "kernel_time_share": share,
        "kernel_ms_per_step": kernel_ms,
        **({"cache": cache_note} if cache_note else {}),
        "clocks": clk,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


def launch_ranks(n: int) -> int:
    """Re-run this command as n ranks of torch.distributed.run on this node
    (rendezvous on 127.0.0.1), bounded by a timeout; rank 0 prints the line."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def fp8_label(mode):
    """The dtype key of the JSON line for a --fp8 mode."""
    if not mode:
        return "bf16"
    gemms = "e4m3 GEMMs but FFN2" if mode.startswith("no-ffn2") else "e4m3 GEMMs"
    return f"bf16 ({gemms}, INT8/e4m3 attention)" if mode.endswith("+attn") else f"bf16 ({gemms})"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cfg-cache", type=float, default=None, metavar="T",
                    help="sample with the CFG cache: steps at noise level <= T reuse the last unconditional velocity")
    ap.add_argument("--attn-cache", type=float, nargs=2, default=None, metavar=("T", "INTERVAL"),
                    help="sample with the attention cache: at noise level <= T recompute the self-attention every "
                         "INTERVAL steps and reuse each block's last output in between")
    ap.add_argument("--cfg-split", action="store_true",
                    help="one video on two GPUs: rank 0 the text row, rank 1 the zeroed-text row (--gpus 2)")
    ap.add_argument("--seq-parallel", action="store_true",
                    help="one video on all GPUs: the blocks under head-sharded (Ulysses) sequence parallelism")
    ap.add_argument("--fp8", nargs="?", const="all", default=None,
                    choices=("all", "no-ffn2", "all+attn", "no-ffn2+attn"),
                    help="the blocks' linear layers as e4m3 GEMMs (per-token / per-channel scales): all six, or all "
                         "but the FFN's second layer (no-ffn2: the FFN hidden stays bf16); +attn: the self-attention "
                         "as the FP8 attention (INT8 Q K^T, e4m3 P V), else bf16")
    ap.add_argument("--ring", type=int, default=1, metavar="R",
                    help="with --seq-parallel: R ring groups (Ulysses inside each group of N/R GPUs, a ring across them)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start the ranks under torch.distributed.run and wait for them
        return launch_ranks(args.gpus)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but the launcher started {world} rank(s); "
                         f"give the launcher --nproc-per-node {args.gpus}\n")
        return 2
    if args.impl == "reference":
        return run_reference(args, rank)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
