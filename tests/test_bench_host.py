"""bench.py's host logic on the CPU: the FLOP count behind the TFLOP/s and
roofline figures (each Linear of the block counted on its own), the DRAM
traffic record's source-hash check, the clock sampler's parsing of the
nvidia-smi lines, and the dtype label of the FP8 modes."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from flow_matching_video_b200 import synth  # noqa: E402


def _linear(n_in, n_out, rows):
    return 2.0 * rows * n_in * n_out


@pytest.mark.parametrize("wl", [synth.STACK_480P81, synth.STACK_480P81_T2V, synth.WIDE_720P81])
def test_step_flops_counts_every_linear_and_attention(wl):
    """One CFG step = batch x (blocks x block + patch embedding + head); the
    cross-attention's K/V projections of the context run once per video and
    are not part of a step."""
    d = wl.dims
    L, D, F = d.L, d.D, d.ffn
    block = (_linear(D, 3 * D, L)                      # q | k | v
             + _linear(D, D, L)                        # self-attention output
             + _linear(D, D, L)                        # cross-attention query
             + _linear(D, D, L)                        # cross-attention output
             + _linear(D, F, L) + _linear(F, D, L)     # feed-forward
             + 2 * (2.0 * L * L * D)                   # S = Q K^T and O = P V, all heads
             + 2 * (2.0 * L * (d.n_img + d.n_txt) * D))  # the same over the image and text keys
    extra = _linear(d.patch_k, D, L) + _linear(D, 16 * 1 * 2 * 2, L)   # patch embedding, head
    assert bench.step_flops(d, 2) == pytest.approx(2 * (d.blocks * block + extra), rel=1e-12)
    f = bench.block_flops(d)
    assert f["attn_self"] == pytest.approx(4.0 * L * L * D, rel=1e-12)


def test_traffic_record_applies_only_to_the_captured_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"the captured kernel")
    sha = hashlib.sha256(b"the captured kernel").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(
        json.dumps({"attn_self": {"source_sha": sha, "bytes_per_launch": 123.0}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("attn_self", str(src)) == 123.0
    assert bench.traffic_for("attn_cross", str(src)) is None
    src.write_bytes(b"the kernel, changed since")
    assert bench.traffic_for("attn_self", str(src)) is None


def test_committed_traffic_records_are_well_formed():
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert rec
    for name, r in rec.items():
        assert len(r["source_sha"]) == 16 and int(r["source_sha"], 16) >= 0, name
        assert r["bytes_per_launch"] > 0, name


class _Done:
    def terminate(self):
        pass

    def wait(self):
        return 0


def test_clock_sampler_takes_the_median_and_the_active_reasons(tmp_path):
    c = bench.Clocks()
    c.f = open(tmp_path / "clocks.csv", "w+")
    c.f.write("0, 1500, 1965, 880.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
              "0, 1560, 1965, 901.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
              "0, [N/A], 1965, 0.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
              "a short line\n"
              "0, 1530, 1965, 899.9, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    c.proc = _Done()
    out = c.stop()
    assert out["sm_mhz"] == 1530.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3
    assert not os.path.exists(tmp_path / "clocks.csv")


def test_clock_sampler_without_nvidia_smi():
    c = bench.Clocks()
    c.proc = None
    assert c.stop() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}


@pytest.mark.parametrize("mode,label", [
    (None, "bf16"),
    ("all", "bf16 (e4m3 GEMMs)"),
    ("no-ffn2", "bf16 (e4m3 GEMMs but FFN2)"),
    ("all+attn", "bf16 (e4m3 GEMMs, INT8/e4m3 attention)"),
    ("no-ffn2+attn", "bf16 (e4m3 GEMMs but FFN2, INT8/e4m3 attention)"),
])
def test_fp8_modes_are_named_in_the_dtype_key(mode, label):
    assert bench.fp8_label(mode) == label
