"""Kernel-by-kernel parity of the CUDA path against the CPU oracle.

Each test calls one libwd entry point through the C ABI and compares every
output element with the oracle on the same seeded inputs.  Tolerances:
the path's stated bars, max |gpu - oracle| / rms(oracle) <= 1e-4 for fp32
arithmetic and <= 2e-2 for bf16 storage, and, where a kernel stores a
rounded value, an elementwise bound derived from the arithmetic (half a bf16
ulp per store plus the fp32 accumulation bound); exact for the 0/1 mask and
copies.
"""
import numpy as np
import pytest
import torch

from oracle import wan_oracle as O
from flow_matching_video_b200 import synth

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def wd():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from flow_matching_video_b200 import build
    build.build()
    from flow_matching_video_b200 import wd as _wd
    return _wd


def rel(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu))
    return float(np.abs(gpu - ref).max() / max(np.sqrt((ref * ref).mean()), 1e-30))


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda", dtype)


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def bf(a):
    return O.bf16(a)


# ------------------------------------------------------------------ Euler / CFG
@pytest.mark.parametrize("n", [1, 7, 4096 + 3, 16 * 21 * 60 * 104])
def test_euler_cfg(wd, n):
    rng = np.random.default_rng(n)
    x, vc, vu = (rng.standard_normal(n).astype(np.float32) for _ in range(3))
    gx = dev(x)
    wd.wd_euler_cfg_step(gx, dev(vc), dev(vu), 5.0, 1 / 12)
    wd.wd_check()
    assert rel(host(gx), O.euler_cfg_step(x, vc, vu, 5.0, 1 / 12)) < 1e-6
    gx = dev(x)
    wd.wd_euler_cfg_step(gx, dev(vc), None, 5.0, 0.5)
    wd.wd_check()
    assert rel(host(gx), O.euler_cfg_step(x, vc, None, 5.0, 0.5)) < 1e-6


def test_euler_exact_velocity_lands_on_data(wd):
    rng = np.random.default_rng(3)
    x0, x1 = rng.standard_normal((2, 16, 3, 8, 8)).astype(np.float32)
    v = (x1.astype(np.float64) - x0).astype(np.float32)
    gx = dev(x0)
    wd.wd_euler_cfg_step(gx, dev(v), dev(v), 5.0, 1.0)
    wd.wd_check()
    np.testing.assert_allclose(host(gx), x1, atol=1e-6)


# ------------------------------------------------------------------ conditioning
@pytest.mark.parametrize("known", [None, [0], [0, 80], [5, 17, 80]])
def test_build_cond_y_exact(wd, known):
    d = synth.Dims(D=128, heads=4, ffn=512, blocks=1, T=21, H=6, W=10, n_txt=4, c_txt=8, n_img=2, c_img=8,
                   dtype="f32")
    img = np.random.default_rng(1).standard_normal((16, 21, 6, 10)).astype(np.float32)
    y = torch.empty((20, 21, 6, 10), device="cuda")
    wd.wd_build_cond_y(wd.make_dims(d), dev(img), y, known)
    wd.wd_check()
    want = O.build_cond_y(img, known or (0,))
    np.testing.assert_array_equal(host(y), want)


# ------------------------------------------------------------------ time MLP
@pytest.mark.parametrize("wl", [synth.TINY, synth.STACK_480P81], ids=lambda w: w.name)
@pytest.mark.parametrize("tau", [1000.0, 437.5, 0.0])
def test_time_mod(wd, wl, tau):
    w = synth.model_weights(wl, blocks=[])
    D = wl.dims.D
    tw = {k: dev(w[k]) for k in ("t1.w", "t1.b", "t2.w", "t2.b", "tp.w", "tp.b")}
    st = wd.wd_time_weights(*(tw[k].data_ptr() for k in ("t1.w", "t1.b", "t2.w", "t2.b", "tp.w", "tp.b")))
    e, e0 = torch.empty(D, device="cuda"), torch.empty((6, D), device="cuda")
    wd.wd_time_mod(wd.make_dims(wl.dims), st, tau, e, e0)
    wd.wd_check()
    re, re0 = O.time_mod(w, tau, D)
    assert rel(host(e), re) < TOL_F32
    assert rel(host(e0), re0) < TOL_F32


# ------------------------------------------------------------------ GEMM with fused epilogues
GEMM_SHAPES = [(300, 192, 72), (128, 256, 64), (1000, 384, 1536), (257, 64, 144), (4096, 4608, 1536),
               (2000, 8960, 1536), (1500, 1536, 8960)]


U32 = 2.0 ** -24          # fp32 unit roundoff
BF16_HALF_ULP = 2.0 ** -8 # bf16 round-to-nearest: |round(v) - v| <= 2^-8 |v|
F16_HALF_ULP = 2.0 ** -11 # IEEE half, normal range: |round(v) - v| <= 2^-11 |v|
F16_SUB = 2.0 ** -25      # IEEE half below 2^-14: |round(v) - v| <= 2^-25


def _gemm_case(wd, dtype, M, N, K, epi, seed=0):
    """Run one GEMM and return (got, exact, bound): an elementwise error bound
    derived from the arithmetic.  Accumulating K products in fp32 in any order
    errs by at most K*u*sum|a_k b_k| (u = 2^-24; doubled to allow truncating
    adders); a bf16 store adds at most half an ulp, 2^-8 |v| (an IEEE half
    store 2^-11 |v|, or 2^-25 below 2^-14); GELU has slope below 1.13."""
    rng = np.random.default_rng(seed + M + N + K + epi)
    A = rng.standard_normal((M, K)).astype(np.float32)
    B = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    bias = rng.standard_normal(N).astype(np.float32) * 0.1
    ga, gb = rng.standard_normal(N).astype(np.float32), rng.standard_normal(N).astype(np.float32) * 0.1
    is_bf = dtype == wd.WD_BF16
    if is_bf:
        A, B = bf(A).astype(np.float32), bf(B).astype(np.float32)
    tdt = torch.bfloat16 if is_bf else torch.float32
    acc = O.linear(A, B, bias)
    acc_err = 2.0 * K * U32 * (np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64)).T + np.abs(bias))
    if epi == wd.EPI_RESID:
        X0 = rng.standard_normal((M, N)).astype(np.float32)
        out = dev(X0)
        g = ga.astype(np.float64) + gb
        want = X0 + g * acc
        bound = np.abs(g) * acc_err + 2 * U32 * (np.abs(X0) + np.abs(g * acc))
    else:
        odt = {wd.EPI_F32: torch.float32, wd.EPI_STORE_F16: torch.float16}.get(epi, tdt)
        out = torch.empty((M, N), device="cuda", dtype=odt)
        if epi == wd.EPI_GELU:
            want = O.gelu(acc)
            bound = 1.13 * acc_err + 1e-6 * (np.abs(want) + 1.0)
        else:
            want = acc
            bound = acc_err + U32 * np.abs(want)
        if epi == wd.EPI_STORE_F16:
            bound = bound * (1 + F16_HALF_ULP) + F16_HALF_ULP * np.abs(want) + F16_SUB
        elif epi != wd.EPI_F32 and is_bf:
            bound = bound * (1 + BF16_HALF_ULP) + BF16_HALF_ULP * np.abs(want)
    wd.wd_gemm(dtype, M, N, K, dev(A, tdt), dev(B, tdt), dev(bias), epi, out,
               dev(ga) if epi == wd.EPI_RESID else None, dev(gb) if epi == wd.EPI_RESID else None)
    wd.wd_check()
    return host(out), want, bound


def assert_within(got, want, bound):
    err = np.abs(got - want)
    bad = err > bound
    assert np.all(np.isfinite(got))
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; worst excess {float((err - bound).max())}"


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_gemm_bf16_tensor_cores(wd, M, N, K, epi):
    got, want, bound = _gemm_case(wd, wd.WD_BF16, M, N, K, epi)
    assert_within(got, want, bound)
    if epi in (2, 3):
        assert rel(got, want) < TOL_F32 * max(1.0, (K / 1536) ** 0.5)


@pytest.mark.parametrize("M,N,K", [(300, 192, 72), (97, 64, 144), (513, 128, 300)])
@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_gemm_f32_cuda_cores(wd, M, N, K, epi):
    got, want, bound = _gemm_case(wd, wd.WD_F32, M, N, K, epi)
    assert_within(got, want, bound)
    assert rel(got, want) < TOL_F32


@pytest.mark.parametrize("M,N,K", [(2 * 512, 1536, 1536), (257, 5120, 5120), (97, 64, 144)])
def test_gemm_bf16_half_store(wd, M, N, K):
    """Epilogue 5: the cross-attention operands stored as IEEE half."""
    got, want, bound = _gemm_case(wd, wd.WD_BF16, M, N, K, wd.EPI_STORE_F16)
    assert_within(got, want, bound)


@pytest.mark.parametrize("epi", [0, 5])
def test_gemm_bf16_simt_reference_kernel(wd, epi):
    wd.wd_set_debug_flags(1)
    try:
        got, want, bound = _gemm_case(wd, wd.WD_BF16, 300, 192, 72, epi)
    finally:
        wd.wd_set_debug_flags(0)
    assert_within(got, want, bound)


# ------------------------------------------------------------------ attention
ATTN_CASES = [  # batch, Lq, heads, dh, n1, shared1, n2, shared2
    (1, 200, 2, 128, 200, 0, 0, 0),
    (2, 300, 2, 128, 300, 0, 0, 0),
    (1, 100, 1, 128, 100, 0, 0, 0),
    (1, 2048, 1, 128, 2048, 0, 0, 0),
    (2, 130, 3, 128, 257, 1, 512, 0),
    (1, 513, 1, 128, 1, 1, 0, 0),
    (1, 64, 2, 64, 9, 1, 16, 0),
    (2, 32, 4, 32, 32, 0, 0, 0),
    (1, 1000, 2, 128, 1000, 0, 0, 0),
]


def _attn_case(wd, dtype, b, Lq, h, dh, n1, s1, n2, s2, seed=0):
    """Run one attention and return (got, exact, bound).  The exact value is
    the oracle's attention on the same (representable) inputs, unrounded.
    Bound: a bf16 output store errs by at most 2^-8 |o|; probabilities stored
    in the operand type before the P V product err by at most u p each
    (u = 2^-8 for bf16, 2^-11 for IEEE half), which moves o by at most
    u * softmax(q k^T) |v| (doubled for the fp32 sums and ex2)."""
    rng = np.random.default_rng(seed + Lq + n1 + n2 + dh)
    D = h * dh
    q = rng.standard_normal((b, Lq, D)).astype(np.float32)
    k1 = rng.standard_normal(((1 if s1 else b), n1, D)).astype(np.float32)
    v1 = rng.standard_normal(((1 if s1 else b), n1, D)).astype(np.float32)
    k2 = v2 = None
    if n2:
        k2 = rng.standard_normal(((1 if s2 else b), n2, D)).astype(np.float32)
        v2 = rng.standard_normal(((1 if s2 else b), n2, D)).astype(np.float32)
    is_bf, is_half = dtype == wd.WD_BF16, dtype == wd.WD_F16
    rnd = bf if is_bf else (lambda a: a.astype(np.float16).astype(np.float32)) if is_half else (lambda a: a)
    q, k1, v1 = rnd(q), rnd(k1), rnd(v1)
    if n2:
        k2, v2 = rnd(k2), rnd(v2)
    tdt = torch.bfloat16 if is_bf else torch.float16 if is_half else torch.float32
    o = torch.empty((b, Lq, D), device="cuda", dtype=torch.bfloat16 if is_half else tdt)
    wd.wd_attention(dtype, b, Lq, h, dh, dev(q, tdt), dev(k1, tdt), dev(v1, tdt), n1, s1, o,
                    dev(k2, tdt) if n2 else None, dev(v2, tdt) if n2 else None, n2, s2)
    wd.wd_check()
    want = np.empty((b, Lq, D))
    pv_abs = np.empty((b, Lq, D))
    for bb in range(b):
        qq = q[bb].reshape(Lq, h, dh)
        segs = [(k1[0 if s1 else bb], v1[0 if s1 else bb], n1)]
        if n2:
            segs.append((k2[0 if s2 else bb], v2[0 if s2 else bb], n2))
        r = 0.0
        ra = 0.0
        for kk, vv, n in segs:
            r = r + O.attention(qq, kk.reshape(n, h, dh), vv.reshape(n, h, dh))
            ra = ra + O.attention(qq, kk.reshape(n, h, dh), np.abs(vv).reshape(n, h, dh))
        want[bb] = r.reshape(Lq, D)
        pv_abs[bb] = ra.reshape(Lq, D)
    if is_bf or is_half:
        u_p = BF16_HALF_ULP if is_bf else F16_HALF_ULP
        bound = BF16_HALF_ULP * np.abs(want) + 2 * u_p * pv_abs + 1e-6
    else:
        bound = 1e-5 * (np.abs(want) + pv_abs)
    return host(o), want, bound


@pytest.mark.parametrize("case", ATTN_CASES)
def test_attention_bf16(wd, case):
    got, want, bound = _attn_case(wd, wd.WD_BF16, *case)
    assert_within(got, want, bound)


@pytest.mark.parametrize("case", ATTN_CASES)
def test_attention_half_operands(wd, case):
    """IEEE half q/k/v (and P), bf16 output: the bf16 model's cross-attention."""
    got, want, bound = _attn_case(wd, wd.WD_F16, *case)
    assert_within(got, want, bound)


@pytest.mark.parametrize("case", ATTN_CASES)
def test_attention_f32(wd, case):
    got, want, bound = _attn_case(wd, wd.WD_F32, *case)
    assert_within(got, want, bound)
    assert rel(got, want) < TOL_F32


@pytest.mark.parametrize("half", [0, 1])
def test_attention_bf16_simt_reference_kernel(wd, half):
    wd.wd_set_debug_flags(2)
    try:
        got, want, bound = _attn_case(wd, wd.WD_F16 if half else wd.WD_BF16, 2, 130, 3, 128, 257, 1, 512, 0)
    finally:
        wd.wd_set_debug_flags(0)
    assert_within(got, want, bound)


# ------------------------------------------------------------------ FP8 building blocks ("Wan（通义万相）..." 5.3)
def _e4m3_bytes(vals):
    """e4m3 values (float64, exactly representable) -> their one-byte codes."""
    return torch.from_numpy(np.ascontiguousarray(vals)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# one warp per row (K <= 2048), eight warps per row (K <= 16384) and the two-pass kernel (longer rows, fp32),
# each at its boundaries and with row counts that leave a block part-filled
@pytest.mark.parametrize("rows,K,dtype", [(257, 1536, "bf16"), (3, 8, "bf16"), (5, 2048, "bf16"), (130, 8960, "bf16"),
                                          (7, 2056, "bf16"), (9, 16384, "bf16"), (2, 16392, "bf16"), (64, 136, "f32")])
def test_quant_rows_e4m3_bit_exact(wd, rows, K, dtype):
    rng = np.random.default_rng(rows + K)
    x = (rng.standard_normal((rows, K)) * np.exp(rng.uniform(-4, 4, (rows, 1)))).astype(np.float32)
    x[min(1, rows - 1)] = 0.0                                    # an all-zero row
    if dtype == "bf16":
        x = bf(x).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    wd.wd_quant_rows_e4m3(wd.WD_BF16 if dtype == "bf16" else wd.WD_F32, rows, K, dev(x, tdt), q, s)
    wd.wd_check()
    want_q, want_s = O.quant_rows_e4m3(x)
    np.testing.assert_array_equal(s.cpu().numpy(), want_s)
    np.testing.assert_array_equal(q.cpu().numpy(), _e4m3_bytes(want_q))


FP8_SHAPES = [(300, 256, 128), (2000, 1536, 1536), (1000, 8960, 1536), (513, 1536, 8960), (129, 4608, 64)]


@pytest.mark.parametrize("M,N,K", FP8_SHAPES)
@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_gemm_fp8_tensor_cores(wd, M, N, K, epi):
    """Operands quantised on the GPU (checked against the oracle's codes), then the
    e4m3 GEMM against the oracle's scaled product of the same codes.  Bound: the
    products of two e4m3 codes are exact in fp32, so the accumulation errs by at
    most 2K u sum|qa qb|; scaling and bias add 3 u |v|; a bf16 store 2^-8 |v|."""
    rng = np.random.default_rng(M + N + K + epi)
    A = bf(rng.standard_normal((M, K))).astype(np.float32)
    B = bf(rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    bias = rng.standard_normal(N).astype(np.float32) * 0.1
    ga, gb = rng.standard_normal(N).astype(np.float32), rng.standard_normal(N).astype(np.float32) * 0.1
    qa, sa = (torch.empty((M, K), dtype=torch.uint8, device="cuda"), torch.empty(M, device="cuda"))
    qb, sb = (torch.empty((N, K), dtype=torch.uint8, device="cuda"), torch.empty(N, device="cuda"))
    wd.wd_quant_rows_e4m3(wd.WD_BF16, M, K, dev(A, torch.bfloat16), qa, sa)
    wd.wd_quant_rows_e4m3(wd.WD_BF16, N, K, dev(B, torch.bfloat16), qb, sb)
    oqa, osa = O.quant_rows_e4m3(A)
    oqb, osb = O.quant_rows_e4m3(B)
    np.testing.assert_array_equal(qa.cpu().numpy(), _e4m3_bytes(oqa))
    np.testing.assert_array_equal(qb.cpu().numpy(), _e4m3_bytes(oqb))
    v = O.gemm_fp8(oqa, osa, oqb, osb, bias)
    s2 = np.abs(osa.astype(np.float64))[:, None] * np.abs(osb.astype(np.float64))[None, :]
    acc_err = 2.0 * K * U32 * (np.abs(oqa) @ np.abs(oqb).T) * s2 + 3 * U32 * (np.abs(v) + np.abs(bias))
    if epi == 3:
        X0 = rng.standard_normal((M, N)).astype(np.float32)
        out = dev(X0)
        g = ga.astype(np.float64) + gb
        want = X0 + g * v
        bound = np.abs(g) * acc_err + 2 * U32 * (np.abs(X0) + np.abs(g * v))
    else:
        out = torch.empty((M, N), device="cuda", dtype=torch.float32 if epi == 2 else torch.bfloat16)
        want = O.gelu(v) if epi == 1 else v
        bound = (1.13 if epi == 1 else 1.0) * acc_err + U32 * np.abs(want) + 1e-6 * (epi == 1)
        if epi != 2:
            bound = bound * (1 + BF16_HALF_ULP) + BF16_HALF_ULP * np.abs(want)
    wd.wd_gemm_fp8(M, N, K, qa, sa, qb, sb, dev(bias), epi, out, dev(ga) if epi == 3 else None,
                   dev(gb) if epi == 3 else None)
    wd.wd_check()
    assert_within(host(out), want, bound)


# ------------------------------------------------------------------ the softmax's 2^x and the bounded waits
def test_exp2_fma_within_its_stated_bound(wd):
    """The FMA-pipe 2^x of the attention softmax, on a dense grid over
    [-130, 0] plus every half-integer (where the range reduction's rounding
    switches the integer part) and its float32 neighbours: relative error at
    most 7.5e-5 against float64 2^x, the bound its polynomial was fitted to;
    inputs below -125 give 2^-125 within the same bound.  Its packed
    two-lane form must give the same values; the MUFU ex2 and CUDA's exp2f
    are checked beside it."""
    halves = np.arange(-130.0, 0.5, 0.5, dtype=np.float32)
    x = np.concatenate([np.linspace(-130.0, 0.0, 2_000_001, dtype=np.float32), halves,
                        np.nextafter(halves, np.float32(1)), np.nextafter(halves, np.float32(-200)),
                        np.float32([-1e-30, -1e-7, -0.0, -125.0, -125.5, -126.0, -1000.0])]).astype(np.float32)
    gx = dev(x)
    outs = [torch.empty_like(gx) for _ in range(4)]
    wd.wd_test_exp2(gx, *outs)
    wd.wd_check()
    y_fma, y_fma2, y_mufu, y_lib = (o.cpu().numpy().astype(np.float64) for o in outs)
    # the packed two-lane form computes the same function, lane by lane
    np.testing.assert_array_equal(y_fma2, y_fma)
    x64 = x.astype(np.float64)
    ref = np.exp2(np.maximum(x64, -125.0))
    r_fma = np.abs(y_fma / ref - 1.0)
    assert r_fma.max() <= 7.5e-5, (r_fma.max(), x[r_fma.argmax()])
    in_range = x64 >= -125.0
    exact = np.exp2(x64[in_range])
    assert np.abs(y_lib[in_range] / exact - 1.0).max() <= 2.0 ** -22          # exp2f: 2 ulp
    assert np.abs(y_mufu[in_range] / exact - 1.0).max() <= 2.0 ** -20         # far below a bf16 half-ulp
    assert np.abs(y_fma[in_range] / y_lib[in_range] - 1.0).max() <= 7.5e-5 + 2.0 ** -22


def test_gelu_epilogue_within_its_bound(wd):
    """The tensor-core GEMM epilogue's GELU (Abramowitz and Stegun 7.1.26 for
    the normal tail probability), scalar and packed two-lane forms, on a dense
    grid over [-30, 30] plus the sign change and far arguments: within 1e-6 (|GELU(x)| + 1) of the float64
    GELU, the function-error allowance of the GEMM tests, and within 1e-6 of
    the erff form that the CUDA-core path uses; exact 0 at 0, x itself far
    right, 0 far left."""
    from scipy.special import erfc
    x = np.concatenate([np.linspace(-30.0, 30.0, 4_000_001, dtype=np.float32),
                        np.float32([0.0, -0.0, 1e-30, -1e-30, 1e-7, -1e-7, 50.0, -50.0, 1e4, -1e4])])
    gx = dev(x)
    y_as, y_as2, y_erf = torch.empty_like(gx), torch.empty_like(gx), torch.empty_like(gx)
    wd.wd_test_gelu(gx, y_as, y_as2, y_erf)
    wd.wd_check()
    ya, ya2, ye = (t.cpu().numpy().astype(np.float64) for t in (y_as, y_as2, y_erf))
    # the packed two-lane form (the one the epilogue runs) computes the same function, lane by lane
    np.testing.assert_array_equal(ya2, ya)
    x64 = x.astype(np.float64)
    exact = 0.5 * x64 * erfc(-x64 / np.sqrt(2.0))
    err = np.abs(ya - exact)
    assert np.all(err <= 1e-6 * (np.abs(exact) + 1.0)), (err.max(), x[err.argmax()])
    assert np.abs(ya - ye).max() <= 1e-6
    assert ya[x == 0.0].max() == 0.0 and ya[x == 0.0].min() == 0.0
    far = np.abs(x64) >= 50.0
    np.testing.assert_array_equal(ya[far], np.where(x64[far] > 0, x64[far], 0.0))


def test_bounded_wait_runs_out_reports_and_recovers(wd):
    """A wait that nothing completes, with a 1 ms limit: the kernel returns,
    wd_check reports WD_ERR_TIMEOUT with the site and clears the error word,
    the next wd_check is clean, and the library keeps working (a GEMM then
    meets its bound)."""
    out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    wd.wd_check()
    wd.wd_test_wait_timeout(1_000_000, 0x9A1, out)
    assert wd.wd_check_status() == 7
    assert "0x9a1" in wd.wd_last_error()
    assert int(out.item()) == 0
    assert wd.wd_check_status() == 0
    got, want, bound = _gemm_case(wd, wd.WD_BF16, 300, 192, 72, 3)
    assert_within(got, want, bound)


# ------------------------------------------------------------------ attention over key parts: log-sum-exp and merge
@pytest.mark.parametrize("dtype,dh,Lq,n", [("bf16", 128, 300, 1000), ("bf16", 128, 2048, 2048), ("f32", 32, 130, 200)])
def test_attention_lse_and_merge_over_key_parts(wd, dtype, dh, Lq, n):
    """wd_attention_lse returns each row's log-sum-exp (log2 units) of the
    scaled scores; merging the attentions over three disjoint key parts by
    log-sum-exp (wd_attention_merge) gives the attention over all keys.
    Bounds: the log-sum-exp within 2e-4 (fp32 sums of 2^x, each within the
    FMA-pipe 2^x's 7.5e-5); the merged output within the attention bound of
    each part (its weights sum to 1) plus the rounding of the output."""
    is_bf = dtype == "bf16"
    dt = wd.WD_BF16 if is_bf else wd.WD_F32
    tdt = torch.bfloat16 if is_bf else torch.float32
    rng = np.random.default_rng(Lq + n + dh)
    B, h = 2, 2
    q, k, v = (rng.standard_normal((B, m, h * dh)).astype(np.float32) for m in (Lq, n, n))
    if is_bf:
        q, k, v = (bf(a).astype(np.float32) for a in (q, k, v))
    qd, kd, vd = dev(q, tdt), dev(k, tdt), dev(v, tdt)
    # exact attention and log-sum-exp per (batch, head, row)
    qa, ka, va = (a.astype(np.float64).reshape(B, -1, h, dh) for a in (q, k, v))
    s = np.einsum("bmhd,bnhd->bhmn", qa, ka) / np.sqrt(dh)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    want_o = np.einsum("bhmn,bnhd->bmhd", p, va).reshape(B, Lq, h * dh)
    sm = s.max(-1, keepdims=True)
    want_lse = (sm[..., 0] + np.log(np.exp(s - sm).sum(-1))) / np.log(2.0)
    o = torch.empty((B, Lq, h * dh), device="cuda", dtype=tdt)
    lse = torch.empty((B, h, Lq), device="cuda")
    wd.wd_attention_lse(dt, B, Lq, h, dh, qd, kd, vd, n, 0, o, lse)
    wd.wd_check()
    assert np.abs(host(lse) - want_lse).max() <= 2e-4
    # three parts of the keys, merged in turn
    o_run = torch.empty((B, Lq, h * dh), device="cuda")
    lse_run = torch.empty((B, h, Lq), device="cuda")
    out = torch.empty((B, Lq, h * dh), device="cuda", dtype=tdt)
    cuts = [0, n // 5, (3 * n) // 4, n]
    for j in range(3):
        a, b_ = cuts[j], cuts[j + 1]
        op = torch.empty((B, Lq, h * dh), device="cuda", dtype=tdt)
        lp = torch.empty((B, h, Lq), device="cuda")
        wd.wd_attention_lse(dt, B, Lq, h, dh, qd, kd[:, a:b_].contiguous(), vd[:, a:b_].contiguous(), b_ - a, 0, op, lp)
        wd.wd_attention_merge(dt, B, Lq, h, dh, o_run, lse_run, op, lp, j == 0, out if j == 2 else None)
    wd.wd_check()
    assert np.abs(host(lse_run) - want_lse).max() <= 3e-4
    u_out = BF16_HALF_ULP if is_bf else 2 * U32
    vbar = np.einsum("bhmn,bnhd->bmhd", p, np.abs(va)).reshape(B, Lq, h * dh)
    bound = 2 * u_out * np.abs(want_o) + (4 * BF16_HALF_ULP if is_bf else 1e-5) * vbar + 1e-6
    assert_within(host(out), want_o, bound)


@pytest.mark.parametrize("seed", [0, 1])
def test_attention_bf16_reference_moves(wd, seed):
    """Key groups whose scores rise far above every earlier key block's (by
    more than 58 in log2 units for most rows), so the online softmax must move
    its reference and rescale O and the row sum deep into the row: head 0,
    keys 300-309 scaled by 40 (in key block 2); head 1, keys 300-309 scaled
    by 4 (a rise within the lazy threshold for some rows) and keys 600-609 by
    40 (the second half of block 4).  Output and log-sum-exp against the
    exact attention, with the bounds of the other attention tests; the
    log-sum-exp bound adds the fp32 accumulation bound of the scores
    (dh * 2^-24 * sum |q_i k_i|)."""
    B, Lq, h, dh, n = 1, 300, 2, 128, 640
    rng = np.random.default_rng(500 + seed)
    q, k, v = (rng.standard_normal((B, m, h * dh)) for m in (Lq, n, n))
    k[:, 300:310, :dh] *= 40.0
    k[:, 300:310, dh:] *= 4.0
    k[:, 600:610, dh:] *= 40.0
    q, k, v = (bf(a.astype(np.float32)).astype(np.float32) for a in (q, k, v))
    qa, ka, va = (a.astype(np.float64).reshape(B, -1, h, dh) for a in (q, k, v))
    s = np.einsum("bmhd,bnhd->bhmn", qa, ka) / np.sqrt(dh)
    sm = s.max(-1, keepdims=True)
    p = np.exp(s - sm)
    want_lse = (sm[..., 0] + np.log(p.sum(-1))) / np.log(2.0)
    p /= p.sum(-1, keepdims=True)
    want = np.einsum("bhmn,bnhd->bmhd", p, va).reshape(B, Lq, h * dh)
    pv_abs = np.einsum("bhmn,bnhd->bmhd", p, np.abs(va)).reshape(B, Lq, h * dh)
    # the rows really jump: by more than 58 (log2 units) above all earlier keys, in both heads
    s2 = s / np.log(2.0)
    assert (s2[0, 0, :, 300:310].max(-1) - s2[0, 0, :, :256].max(-1) > 58).mean() > 0.5
    assert (s2[0, 1, :, 600:610].max(-1) - s2[0, 1, :, :512].max(-1) > 58).mean() > 0.5
    o = torch.empty((B, Lq, h * dh), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((B, h, Lq), device="cuda")
    wd.wd_attention_lse(wd.WD_BF16, B, Lq, h, dh, dev(q, torch.bfloat16), dev(k, torch.bfloat16),
                        dev(v, torch.bfloat16), n, 0, o, lse)
    wd.wd_check()
    bound = BF16_HALF_ULP * np.abs(want) + 2 * BF16_HALF_ULP * pv_abs + 1e-6
    assert_within(host(o), want, bound)
    acc = dh * 2.0 ** -24 * np.einsum("bmhd,bnhd->bhmn", np.abs(qa), np.abs(ka)).max(-1) / np.sqrt(dh) / np.log(2.0)
    assert np.all(np.abs(host(lse) - want_lse) <= 2e-4 + acc)


# ------------------------------------------------------------------ FP8 attention ("Wan（通义万相）..." 5.3)
# (batch, L, heads): ragged small cases, and the 480x832x81 block's self-attention (L = 32760, 12 heads, batch 2)
ATTN8_CASES = [(2, 300, 2), (1, 129, 1), (2, 32760, 12)]


def _qkv8(batch, L, heads, seed):
    """A fused bf16 q|k|v buffer [batch, L, 3D] (host float32 copy, device bf16)
    with per-channel spreads, so that the rows, key blocks and value channels
    all get different scales."""
    rng = np.random.default_rng(seed)
    D = heads * 128
    x = rng.standard_normal((batch, L, 3 * D), dtype=np.float32)
    x[..., :2 * D] *= rng.uniform(0.5, 2.0, 2 * D).astype(np.float32)
    x[..., 2 * D:] *= rng.uniform(0.2, 3.0, D).astype(np.float32)
    x[:, : min(L, 40), :D] *= 3.0                                 # a few large rows of q
    t = torch.from_numpy(x).to(torch.bfloat16)                      # round to nearest even, as O.bf16
    return t.float().numpy(), t.to("cuda")


def _attn8_run(wd, batch, L, heads, seed):
    qh, qd = _qkv8(batch, L, heads, seed)
    D = heads * 128
    lay = wd.wd_attention_fp8_layout(batch, L, L, heads, 128)
    buf = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
    wd.wd_attention_fp8_quantize(batch, L, L, heads, 128, qd, 3 * D, qd[..., D:], qd[..., 2 * D:], 3 * D, buf)
    o = torch.empty((batch, L, D), dtype=torch.bfloat16, device="cuda")
    wd.wd_attention_fp8(batch, L, L, heads, 128, buf, o, D)
    wd.wd_check()
    return qh, lay, buf, o


@pytest.mark.parametrize("batch,L,heads", ATTN8_CASES)
def test_attention_fp8_operands_bit_exact(wd, batch, L, heads):
    """The quantised operands byte for byte against the oracle's quantisers:
    q8 and sq per (row, head), k8 and sk per (128-key block, head), v8t (V
    transposed, e4m3) and sv per (channel, head, batch), the padding keys of
    v8t zero."""
    qh, lay, buf, _ = _attn8_run(wd, batch, L, heads, seed=L + heads)
    D, nb, lkp = heads * 128, (L + 127) // 128, lay.lkp
    cut = lambda off, n, dt: buf[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)
    q8 = cut(lay.q8, batch * L * D, torch.int8).reshape(batch, L, D).cpu().numpy()
    k8 = cut(lay.k8, batch * L * D, torch.int8).reshape(batch, L, D).cpu().numpy()
    sq = cut(lay.sq, batch * heads * L, torch.float32).reshape(batch, heads, L).cpu().numpy()
    sk = cut(lay.sk, batch * heads * nb, torch.float32).reshape(batch, heads, nb).cpu().numpy()
    sv = cut(lay.sv, batch * D, torch.float32).reshape(batch, D).cpu().numpy()
    v8 = cut(lay.v8t, batch * D * lkp, torch.float8_e4m3fn).reshape(batch, heads, 128, lkp).double().cpu().numpy()
    for b in range(batch):
        for h in range(heads):
            cs = slice(h * 128, (h + 1) * 128)
            cq, s_q = O.quant_rows_int8(qh[b, :, cs])
            np.testing.assert_array_equal(q8[b, :, cs], cq)
            np.testing.assert_array_equal(sq[b, h], s_q)
            ck, s_k = O.quant_blocks_int8(qh[b, :, D:][:, cs], 128)
            np.testing.assert_array_equal(k8[b, :, cs], ck)
            np.testing.assert_array_equal(sk[b, h], s_k)
            cv, s_v = O.quant_cols_e4m3(qh[b, :, 2 * D:][:, cs])
            np.testing.assert_array_equal(v8[b, h, :, :L], cv.T)
            np.testing.assert_array_equal(sv[b, cs], s_v)
            assert not v8[b, h, :, L:].any()


@pytest.mark.parametrize("batch,L,heads,n_rows", [(2, 300, 2, None), (1, 129, 1, None), (2, 32760, 12, 64)])
def test_attention_fp8(wd, monkeypatch, batch, L, heads, n_rows):
    """The FP8 attention against the oracle's (the same quantisers, key blocks
    and reference rule) on every row of the small cases and on sampled rows
    plus the ragged tail of the 480p one.  The two differ where the rounding of
    p to e4m3 decides differently: the GPU's 2^x errs by up to 7.5e-5 (FMA
    pipe) and its fp32 logits by a few ulp.  The bar is derived from the oracle
    itself: twice its movement when every p is moved by 1e-4 (seeded), plus
    the rounding of the output to bf16.  Against the exact attention of the
    unquantised inputs the GPU may be no farther than the oracle's FP8
    attention is, plus that bar (the INT8 logits of sharp rows already move the
    oracle by 0.7-0.9 of the output's RMS on these inputs); both are printed."""
    qh, lay, buf, o = _attn8_run(wd, batch, L, heads, seed=7 * L + heads)
    D = heads * 128
    rows = np.arange(L)
    if n_rows is not None:
        rng = np.random.default_rng(L)
        rows = np.unique(np.concatenate([rng.choice(L, n_rows, replace=False), np.arange(L - 40, L), [0, 5]]))
    got = o.float().cpu().numpy()[:, rows].astype(np.float64).reshape(batch, len(rows), heads, 128)
    split = lambda b: (qh[b, rows, :D].reshape(len(rows), heads, 128), qh[b, :, D:2 * D].reshape(L, heads, 128),
                       qh[b, :, 2 * D:].reshape(L, heads, 128))
    want = np.stack([O.attention_fp8(*split(b)) for b in range(batch)])
    prng = np.random.default_rng(99)
    with monkeypatch.context() as m:
        m.setattr(O.np, "exp2", lambda a, _e=np.exp2: _e(a) * (1 + 1e-4 * prng.standard_normal(np.shape(a)))
                  if np.ndim(a) == 2 else _e(a))
        moved = np.stack([O.attention_fp8(*split(b)) for b in range(batch)])
    exact = np.stack([O.attention(*split(b)) for b in range(batch)])
    err, bar = rel(got, want), 2 * rel(moved, want) + rel(bf(want), want)
    e_exact, o_exact = rel(got, exact), rel(want, exact)
    print(f"\n[FP8 attention b={batch} L={L} h={heads}] vs the oracle's FP8 attention {err:.3e} (bar {bar:.3e}); "
          f"vs the exact attention {e_exact:.3e} (the oracle's FP8 attention: {o_exact:.3e})")
    assert err <= bar
    assert e_exact <= o_exact + bar
