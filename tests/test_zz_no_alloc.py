"""wd_patch_embed_noalloc: the patch embedding for callers that cannot
allocate device memory (a host framework that owns the whole device pool and
gives plug-ins no scratch, or a latency-critical loop that must not call
cudaMalloc).  Its scratch is a fixed array inside the library.

Checked through the C ABI against wd_patch_embed (the workspace version) on
two calls in a row with different inputs, at the 480p/81-frame batch-2 size.
Both run the same kernels on the same inputs and differ only in where the
gathered patches sit, so their outputs must agree bit for bit (a tolerance
would let a wrong scratch offset or a stale row through); the output is
prefilled with NaN so that an unwritten row shows.  Plus the size limit.
This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from flow_matching_video_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wd():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from flow_matching_video_b200 import build
    build.build()
    from flow_matching_video_b200 import wd as _wd
    return _wd


def test_noalloc_patch_embed_matches_workspace_version_twice(wd):
    wl = synth.STACK_480P81
    d = wl.dims
    cd = wd.make_dims(d)
    w = synth.model_weights(wl, blocks=[])
    pe_w = torch.from_numpy(w["pe.w"]).cuda().to(torch.bfloat16)
    pe_b = torch.from_numpy(w["pe.b"]).cuda()
    x = synth.inputs(wl)
    y = torch.empty((20, d.T, d.H, d.W), device="cuda")
    wd.wd_build_cond_y(cd, torch.from_numpy(x["img_lat"]).cuda(), y)
    ws = torch.empty(wd.wd_workspace_bytes(cd, wl.batch), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(77)
    for call in range(2):
        x_t = torch.from_numpy(rng.standard_normal((wl.batch, 16, d.T, d.H, d.W)).astype(np.float32)).cuda()
        ref = torch.empty((wl.batch, d.L, d.D), device="cuda")
        got = torch.full((wl.batch, d.L, d.D), float("nan"), device="cuda")
        wd.wd_patch_embed(cd, x_t, y, pe_w, pe_b, wl.batch, ref, ws)
        wd.wd_patch_embed_noalloc(cd, x_t, y, pe_w, pe_b, wl.batch, got)
        wd.wd_check()
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        assert np.all(np.isfinite(g)), f"call {call}: unwritten output"
        assert np.array_equal(g, r), f"call {call}: max |diff| {np.abs(g - r).max()}"


def test_noalloc_patch_embed_rejects_sizes_beyond_the_array(wd):
    d = wd.make_dims(synth.WIDE_720P81.dims)     # 75600 tokens per sample
    lib = wd.lib()
    # batch 3 -> 226800 rows * 144 * 2 bytes > 48 MiB: refused before any launch
    st = lib.wd_patch_embed_noalloc(C.byref(d), 0x1000, 0x2000, 0x3000, 0x4000, 3, 0x5000, None)
    assert st == 5 and "scratch" in wd.wd_last_error()
    # text-to-video patches are 64 wide: the cap is 393216 bf16 rows, so batch 6 (453600 rows) is refused
    import dataclasses
    d = wd.make_dims(dataclasses.replace(synth.WIDE_720P81.dims, n_img=0, c_img=0))
    st = lib.wd_patch_embed_noalloc(C.byref(d), 0x1000, None, 0x3000, 0x4000, 6, 0x5000, None)
    assert st == 5 and "393216" in wd.wd_last_error()
