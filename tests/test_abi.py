"""The C ABI library loads, exports every function include/wd.h declares, and
its host-side logic (sizes, validation) behaves; no GPU is needed.

Validation failures return before any CUDA call, so they can be exercised on
a machine without a GPU.
"""
import ctypes as C
import os
import re

import pytest

from flow_matching_video_b200 import synth
from oracle import wan_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wd():
    from flow_matching_video_b200 import build
    build.build()
    from flow_matching_video_b200 import wd as _wd
    return _wd


def header_functions():
    src = open(os.path.join(ROOT, "include", "wd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wd_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_path():
    fns = header_functions()
    for name in ("wd_build_cond_y", "wd_patch_embed", "wd_time_mod", "wd_block_forward", "wd_unpatchify",
                 "wd_euler_cfg_step", "wd_context_embed", "wd_cross_kv"):
        assert name in fns


def test_every_declared_symbol_is_exported_and_bound(wd):
    lib = wd.lib()
    for name in header_functions():
        assert hasattr(lib, name), name
        assert name in wd.SIGNATURES, name


def test_token_count_and_sizes_match_oracle(wd):
    for wl in synth.WORKLOADS.values():
        d = wd.make_dims(wl.dims)
        F = wl.dims.F_pix
        assert wd.wd_token_count(d) == O.token_count(F, 8 * wl.dims.H, 8 * wl.dims.W) == wl.dims.L
        ws = wd.wd_workspace_bytes(d, wl.batch)
        rows = wl.batch * wl.dims.L
        es = 2 if wl.dims.dtype == "bf16" else 4
        assert ws >= rows * (max(3 * wl.dims.D, wl.dims.ffn) + max(wl.dims.D, 144)) * es
        kv = wd.wd_kv_bytes(d, wl.batch)
        assert kv >= 2 * (wl.dims.n_img + wl.batch * wl.dims.n_txt) * wl.dims.D * es
        assert wd.wd_ctx_bytes(d, wl.batch) >= (wl.batch * wl.dims.n_txt + wl.dims.n_img) * wl.dims.D * es


def test_invalid_dims_rejected(wd):
    d = wd.make_dims(synth.TINY.dims)
    d.heads = 3            # D % heads != 0
    assert wd.wd_workspace_bytes(d, 2) == 0
    d = wd.make_dims(synth.TINY.dims)
    d.H = 7                # odd latent height
    assert wd.wd_workspace_bytes(d, 2) == 0
    d = wd.make_dims(synth.TINY.dims)
    d.dtype = 9
    assert wd.wd_workspace_bytes(d, 2) == 0
    assert wd.wd_workspace_bytes(wd.make_dims(synth.TINY.dims), 0) == 0
    d = wd.make_dims(synth.TINY.dims)
    d.n_img = -1           # negative image token count
    assert wd.wd_workspace_bytes(d, 2) == 0
    d = wd.make_dims(synth.TINY.dims)
    d.c_img = 0            # an image branch needs a CLIP width
    assert wd.wd_workspace_bytes(d, 2) == 0
    # n_img = 0 is the text-to-video model: valid, and its K/V cache holds text only
    d = wd.make_dims(synth.TINY_T2V.dims)
    assert wd.wd_workspace_bytes(d, 2) > 0
    assert wd.wd_kv_bytes(d, 2) == 2 * (2 * 16 * 128 * 4)


def test_patch_embed_needs_y_only_for_image_to_video(wd):
    lib = wd.lib()
    args = (0x1000, None, 0x3000, 0x4000, 2, 0x5000, 0x6000, 16, None)   # y = NULL, tiny workspace
    assert lib.wd_patch_embed(C.byref(wd.make_dims(synth.TINY.dims)), *args) == 1          # WD_ERR_ARG
    assert "y is NULL" in wd.wd_last_error()
    assert lib.wd_patch_embed(C.byref(wd.make_dims(synth.TINY_T2V.dims)), *args) == 5      # workspace check next


def test_null_and_misaligned_pointers_rejected_before_launch(wd):
    lib = wd.lib()
    d = wd.make_dims(synth.TINY.dims)
    # NULL latent -> WD_ERR_ARG
    assert lib.wd_euler_cfg_step(None, None, None, 5.0, 0.5, 16, None) == 1
    assert "NULL" in wd.wd_last_error()
    # misaligned pointers -> WD_ERR_ALIGN, never dereferenced
    assert lib.wd_euler_cfg_step(0x1004, 0x2000, None, 5.0, 0.5, 16, None) == 4
    assert lib.wd_build_cond_y(C.byref(d), 0x1000, None, 0, 0x2008, None) == 4
    # workspace too small -> WD_ERR_WORKSPACE
    hw = wd.wd_head_weights(0x1000, 0x2000, 0x3000)
    assert lib.wd_unpatchify(C.byref(d), C.byref(hw), 0x4000, 2, 0x5000, 0x6000, 0x7000, 16, None) == 5
    # known frame out of range -> WD_ERR_ARG
    kf = (C.c_int * 1)(99)
    assert lib.wd_build_cond_y(C.byref(d), 0x1000, kf, 1, 0x2000, None) == 1
    # bad dtype for the building blocks
    assert lib.wd_gemm(7, 8, 64, 8, 0x1000, 0x2000, None, 0, 0x3000, None, None, None) == 3
    assert lib.wd_attention(7, 1, 8, 1, 32, 0x1000, 0x2000, 0x3000, 8, 0, None, None, 0, 0, 0x4000, None) == 3


def test_product_path_has_no_oracle_import():
    pkg = os.path.join(ROOT, "flow_matching_video_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"(from|import)\s+oracle|wan_oracle|liboracle", src), f


def test_binding_fails_loudly_without_the_library():
    """The product path has no fallback: the binding, run as if it sat in a
    directory without libwd.so, refuses to import (no file is written)."""
    path = os.path.join(ROOT, "flow_matching_video_b200", "wd.py")
    src = open(path, encoding="utf-8").read()
    fake = os.path.join(ROOT, "no_such_directory", "wd.py")
    with pytest.raises(ImportError, match="libwd.so not built"):
        exec(compile(src, path, "exec"), {"__name__": "wd_without_lib", "__file__": fake})


def test_empty_sizes_are_a_no_op_or_rejected_before_launch(wd):
    lib = wd.lib()
    # an empty latent: nothing to update, nothing launched
    assert lib.wd_euler_cfg_step(0x1000, 0x2000, 0x3000, 5.0, 0.5, 0, None) == 0
    # attention without queries or keys, GEMMs without rows: WD_ERR_SHAPE, before any CUDA call
    assert lib.wd_attention(1, 1, 0, 1, 128, 0x1000, 0x2000, 0x3000, 8, 0, None, None, 0, 0, 0x4000, None) == 2
    assert lib.wd_attention(1, 1, 8, 1, 128, 0x1000, 0x2000, 0x3000, 0, 0, None, None, 0, 0, 0x4000, None) == 2
    assert lib.wd_attention(2, 1, 8, 1, 128, 0x1000, 0x2000, 0x3000, 8, 1, 0x5000, 0x6000, 0, 0, 0x4000, None) == 2
    assert lib.wd_gemm(1, 0, 64, 64, 0x1000, 0x2000, None, 0, 0x3000, None, None, None) == 2
    assert lib.wd_gemm_fp8(0, 256, 64, 0x1000, 0x2000, 0x3000, 0x4000, None, 0, 0x5000, None, None, None) == 2
    assert lib.wd_quant_rows_e4m3(1, 0, 64, 0x1000, 0x2000, 0x3000, None) == 2
    assert lib.wd_quant_rows_e4m3(1, 4, 12, 0x1000, 0x2000, 0x3000, None) == 2    # K not a multiple of 8
    # the test-only entries: no values, or a missing output, are refused before any launch
    assert lib.wd_test_gelu(0x1000, 0x2000, 0x3000, 0x4000, 0, None) == 2
    assert lib.wd_test_gelu(0x1000, 0x2000, None, 0x4000, 16, None) == 1
    assert lib.wd_test_exp2(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0, None) == 2
    # the FP8 GEMM's shape rules: N a multiple of 256, scales required
    assert lib.wd_gemm_fp8(8, 128, 64, 0x1000, 0x2000, 0x3000, 0x4000, None, 0, 0x5000, None, None, None) == 2
    assert lib.wd_gemm_fp8(8, 256, 64, 0x1000, None, 0x3000, 0x4000, None, 0, 0x5000, None, None, None) == 1


def test_bf16_model_needs_128_wide_heads(wd):
    """The bf16 model's attention runs on the tensor cores (128-wide heads);
    any other width is refused rather than run on the CUDA cores."""
    lib = wd.lib()
    d = wd.make_dims(synth.SMALL_BF16.dims)
    d.heads = 4                                   # D = 256 -> 64-wide heads
    assert wd.wd_workspace_bytes(d, 2) == 0
    bw = wd.wd_block_weights(*([0x1000] * len(wd.BLOCK_FIELDS)))
    assert lib.wd_block_forward(C.byref(d), C.byref(bw), 0x2000, 0x3000, 2, 0x4000, 0x5000, 1 << 30, None) == 8
    assert "head dim 64" in wd.wd_last_error()
    # the fp32 model keeps its CUDA-core path for any supported width
    d = wd.make_dims(synth.TINY.dims)
    assert wd.wd_workspace_bytes(d, 2) > 0
    assert wd.wd_debug_flags() == 0


def test_fp8_attention_layout_and_refusals(wd):
    """The FP8 attention's operand layout (256-byte aligned regions in order,
    each large enough, the V^T rows padded to 16 keys), and its refusals before
    any CUDA call: head sizes other than 128, empty shapes, short or misaligned
    buffers, misaligned operands."""
    lib = wd.lib()
    B, Lq, Lk, H = 2, 300, 301, 2
    D, nb = H * 128, (Lk + 127) // 128
    lay = wd.wd_attention_fp8_layout(B, Lq, Lk, H, 128)
    assert lay.lkp == 304
    regions = [("q8", B * Lq * D), ("sq", 4 * B * H * Lq), ("k8", B * Lk * D), ("sk", 4 * B * H * nb),
               ("v8t", B * D * lay.lkp), ("sv", 4 * B * D), ("v_amax", 4 * B * D)]
    ends = [getattr(lay, n) for n, _ in regions[1:]] + [lay.bytes]
    for (name, size), end in zip(regions, ends):
        off = getattr(lay, name)
        assert off % 256 == 0 and end - off >= size, name
    out = wd.wd_attn_fp8_layout()
    assert lib.wd_attention_fp8_layout(B, Lq, Lk, H, 64, C.byref(out)) == 8          # dh 64: unsupported
    assert lib.wd_attention_fp8_layout(B, 0, Lk, H, 128, C.byref(out)) == 2          # no queries
    assert lib.wd_attention_fp8_layout(B, Lq, 0, H, 128, C.byref(out)) == 2          # no keys
    q, k, v, buf = 0x10000, 0x20000, 0x30000, 0x100000
    # quantise: buffer too small, then a buffer off its 256-byte alignment, then a misaligned v
    assert lib.wd_attention_fp8_quantize(B, Lq, Lk, H, 128, q, 3 * D, k, v, 3 * D, buf, lay.bytes - 1, None) == 5
    assert lib.wd_attention_fp8_quantize(B, Lq, Lk, H, 128, q, 3 * D, k, v, 3 * D, buf + 16, lay.bytes, None) == 4
    assert lib.wd_attention_fp8_quantize(B, Lq, Lk, H, 128, q, 3 * D, k, v + 8, 3 * D, buf, lay.bytes, None) == 4
    # attention: buffer too small, head size 64
    assert lib.wd_attention_fp8(B, Lq, Lk, H, 128, buf, lay.bytes - 1, 0x200000, D, None) == 5
    assert lib.wd_attention_fp8(B, Lq, Lk, H, 64, buf, lay.bytes, 0x200000, D, None) == 8
