"""ctypes binding of libwd (include/wd.h): argument marshalling only.

Every function here has the name of the C entry point it calls and takes
torch tensors (device memory) where the C function takes device pointers.
All computation happens in the CUDA kernels of libwd.so; when the library is
missing the import fails loudly — there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libwd.so not built ({LIB_PATH}); run `python -m flow_matching_video_b200.build`")
_lib = C.CDLL(LIB_PATH)

WD_F32, WD_BF16, WD_F16 = 0, 1, 2
WD_NORM_LAYER, WD_NORM_RMS = 0, 1
EPI_STORE, EPI_GELU, EPI_F32, EPI_RESID, EPI_STORE_F16 = 0, 1, 2, 3, 5
STATUS = {0: "WD_OK", 1: "WD_ERR_ARG", 2: "WD_ERR_SHAPE", 3: "WD_ERR_DTYPE", 4: "WD_ERR_ALIGN",
          5: "WD_ERR_WORKSPACE", 6: "WD_ERR_CUDA", 7: "WD_ERR_TIMEOUT", 8: "WD_ERR_UNSUPPORTED"}


class WDError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {wd_last_error()}")


class wd_dims(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("D", "heads", "ffn", "blocks", "T", "H", "W", "n_txt", "c_txt",
                                       "n_img", "c_img", "dtype", "norm")] + [("eps", C.c_float)]


def _ptr_struct(name, fields):
    return type(name, (C.Structure,), {"_fields_": [(f, C.c_void_p) for f in fields]})


wd_time_weights = _ptr_struct("wd_time_weights", ["t1_w", "t1_b", "t2_w", "t2_b", "tp_w", "tp_b"])
wd_ctx_weights = _ptr_struct("wd_ctx_weights", ["txt1_w", "txt1_b", "txt2_w", "txt2_b",
                                                "img1_w", "img1_b", "img2_w", "img2_b"])
BLOCK_FIELDS = ["qkv_w", "qkv_b", "g_q", "g_k", "o_w", "o_b", "cn_g", "cn_b", "cq_w", "cq_b", "ck_w", "ck_b",
                "cv_w", "cv_b", "cki_w", "cki_b", "cvi_w", "cvi_b", "co_w", "co_b", "f1_w", "f1_b",
                "f2_w", "f2_b", "mod"]
wd_block_weights = _ptr_struct("wd_block_weights", BLOCK_FIELDS)
wd_head_weights = _ptr_struct("wd_head_weights", ["mod", "w", "b"])
FP8_FIELDS = ["qkv_q", "o_q", "cq_q", "co_q", "f1_q", "f2_q", "qkv_s", "o_s", "cq_s", "co_s", "f1_s", "f2_s"]
wd_block_weights_fp8 = type("wd_block_weights_fp8", (C.Structure,),
                            {"_fields_": [(f, C.c_void_p) for f in FP8_FIELDS] + [("attention_fp8", C.c_int)]})


class wd_attn_fp8_layout(C.Structure):
    _fields_ = [(f, C.c_size_t) for f in ("q8", "sq", "k8", "sk", "v8t", "sv", "v_amax", "bytes")] + \
               [("lkp", C.c_int64)]

# exported symbol -> (restype, argtypes)
_P, _I, _F, _S, _L = C.c_void_p, C.c_int, C.c_float, C.c_size_t, C.c_int64
_PD = C.POINTER(wd_dims)
SIGNATURES = {
    "wd_last_error": (C.c_char_p, []),
    "wd_version": (C.c_char_p, []),
    "wd_check": (_I, [_P]),
    "wd_token_count": (_L, [_PD]),
    "wd_workspace_bytes": (_S, [_PD, _I]),
    "wd_ctx_bytes": (_S, [_PD, _I]),
    "wd_kv_bytes": (_S, [_PD, _I]),
    "wd_build_cond_y": (_I, [_PD, _P, C.POINTER(C.c_int), _I, _P, _P]),
    "wd_context_embed": (_I, [_PD, C.POINTER(wd_ctx_weights), _P, _P, _I, _P, _P]),
    "wd_cross_kv": (_I, [_PD, C.POINTER(wd_block_weights), _P, _I, _P, _P]),
    "wd_time_mod": (_I, [_PD, C.POINTER(wd_time_weights), _F, _P, _P, _P]),
    "wd_patch_embed": (_I, [_PD, _P, _P, _P, _P, _I, _P, _P, _S, _P]),
    "wd_patch_embed_noalloc": (_I, [_PD, _P, _P, _P, _P, _I, _P, _P]),
    "wd_block_forward": (_I, [_PD, C.POINTER(wd_block_weights), _P, _P, _I, _P, _P, _S, _P]),
    "wd_block_qkv": (_I, [_PD, C.POINTER(wd_block_weights), _P, _I, _L, _L, _P, _P, _P, _S, _P]),
    "wd_block_self_attention": (_I, [_PD, _I, _I, _P, _P, _P]),
    "wd_block_post": (_I, [_PD, C.POINTER(wd_block_weights), _P, _P, _I, _L, _P, _P, _P, _S, _P]),
    "wd_workspace_bytes_fp8": (_S, [_PD, _I]),
    "wd_block_forward_fp8": (_I, [_PD, C.POINTER(wd_block_weights), C.POINTER(wd_block_weights_fp8), _P, _P, _I, _P,
                                  _P, _S, _P]),
    "wd_unpatchify": (_I, [_PD, C.POINTER(wd_head_weights), _P, _I, _P, _P, _P, _S, _P]),
    "wd_euler_cfg_step": (_I, [_P, _P, _P, _F, _F, _S, _P]),
    "wd_gemm": (_I, [_I, _I, _I, _I, _P, _P, _P, _I, _P, _P, _P, _P]),
    "wd_attention": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _I, _I, _P, _P, _I, _I, _P, _P]),
    "wd_attention_lse": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _I, _I, _P, _P, _P]),
    "wd_attention_merge": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P]),
    "wd_attention_fp8_layout": (_I, [_I, _L, _L, _I, _I, C.POINTER(wd_attn_fp8_layout)]),
    "wd_attention_fp8_quantize": (_I, [_I, _L, _L, _I, _I, _P, _L, _P, _P, _L, _P, _S, _P]),
    "wd_attention_fp8": (_I, [_I, _L, _L, _I, _I, _P, _S, _P, _L, _P]),
    "wd_quant_rows_e4m3": (_I, [_I, _I, _I, _P, _P, _P, _P]),
    "wd_gemm_fp8": (_I, [_I, _I, _I, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P]),
    "wd_test_exp2": (_I, [_P, _P, _P, _P, _P, _L, _P]),
    "wd_test_gelu": (_I, [_P, _P, _P, _P, _L, _P]),
    "wd_test_wait_timeout": (_I, [C.c_uint64, C.c_uint, _P, _P]),
    "wd_set_debug_flags": (None, [C.c_uint]),
    "wd_debug_flags": (C.c_uint, []),
    "wd_trace_enable": (None, [_I]),
    "wd_trace_read": (_I, [C.POINTER(C.c_int64), C.POINTER(C.c_double)]),
}
KERNEL_CLASSES = ("gemm", "attn_self", "attn_cross", "norm", "qknorm_rope", "euler", "small")
for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def lib():
    return _lib


def _p(t):
    """Device pointer of a tensor (or None)."""
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _ok(status: int, where: str):
    if status != 0:
        raise WDError(status, where)


def make_dims(d) -> wd_dims:
    """wd_dims from a synth.Dims."""
    return wd_dims(d.D, d.heads, d.ffn, d.blocks, d.T, d.H, d.W, d.n_txt, d.c_txt, d.n_img, d.c_img,
                   WD_BF16 if d.dtype == "bf16" else WD_F32, WD_NORM_RMS if d.norm == "rms" else WD_NORM_LAYER,
                   d.eps)


# ------------------------------------------------------------------ entry points
def wd_last_error() -> str:
    return _lib.wd_last_error().decode()


def wd_version() -> str:
    return _lib.wd_version().decode()


def wd_check(stream=None):
    _ok(_lib.wd_check(_stream(stream)), "wd_check")


def wd_token_count(dims: wd_dims) -> int:
    return _lib.wd_token_count(C.byref(dims))


def wd_workspace_bytes(dims: wd_dims, batch: int) -> int:
    return _lib.wd_workspace_bytes(C.byref(dims), batch)


def wd_ctx_bytes(dims: wd_dims, batch: int) -> int:
    return _lib.wd_ctx_bytes(C.byref(dims), batch)


def wd_kv_bytes(dims: wd_dims, batch: int) -> int:
    return _lib.wd_kv_bytes(C.byref(dims), batch)


def wd_build_cond_y(dims, img_lat, y, known_frames=None, stream=None):
    kf, n = None, 0
    if known_frames:
        kf = (C.c_int * len(known_frames))(*known_frames)
        n = len(known_frames)
    _ok(_lib.wd_build_cond_y(C.byref(dims), _p(img_lat), kf, n, _p(y), _stream(stream)), "wd_build_cond_y")


def wd_context_embed(dims, w: wd_ctx_weights, txt, clip, batch, ctx, stream=None):
    _ok(_lib.wd_context_embed(C.byref(dims), C.byref(w), _p(txt), _p(clip), batch, _p(ctx), _stream(stream)),
        "wd_context_embed")


def wd_cross_kv(dims, w: wd_block_weights, ctx, batch, kv, stream=None):
    _ok(_lib.wd_cross_kv(C.byref(dims), C.byref(w), _p(ctx), batch, _p(kv), _stream(stream)), "wd_cross_kv")


def wd_time_mod(dims, w: wd_time_weights, tau: float, e, e0, stream=None):
    _ok(_lib.wd_time_mod(C.byref(dims), C.byref(w), float(tau), _p(e), _p(e0), _stream(stream)), "wd_time_mod")


def wd_patch_embed(dims, x_t, y, w, b, batch, X, ws, stream=None):
    _ok(_lib.wd_patch_embed(C.byref(dims), _p(x_t), _p(y), _p(w), _p(b), batch, _p(X), _p(ws), ws.numel() * ws.element_size(),
                            _stream(stream)), "wd_patch_embed")


def wd_patch_embed_noalloc(dims, x_t, y, w, b, batch, X, stream=None):
    """wd_patch_embed without a workspace: the library's fixed scratch array
    is used instead (for callers that cannot allocate device memory)."""
    _ok(_lib.wd_patch_embed_noalloc(C.byref(dims), _p(x_t), _p(y), _p(w), _p(b), batch, _p(X), _stream(stream)),
        "wd_patch_embed_noalloc")


def wd_block_forward(dims, w: wd_block_weights, e0, kv, batch, X, ws, stream=None):
    _ok(_lib.wd_block_forward(C.byref(dims), C.byref(w), _p(e0), _p(kv), batch, _p(X), _p(ws),
                              ws.numel() * ws.element_size(), _stream(stream)), "wd_block_forward")


def wd_block_qkv(dims, w: wd_block_weights, e0, batch, tok0, n_tok, X, qkv, ws, stream=None):
    _ok(_lib.wd_block_qkv(C.byref(dims), C.byref(w), _p(e0), batch, tok0, n_tok, _p(X), _p(qkv), _p(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "wd_block_qkv")


def wd_block_self_attention(dims, batch, heads, qkv, o, stream=None):
    _ok(_lib.wd_block_self_attention(C.byref(dims), batch, heads, _p(qkv), _p(o), _stream(stream)),
        "wd_block_self_attention")


def wd_block_post(dims, w: wd_block_weights, e0, kv, batch, n_tok, o, X, ws, stream=None):
    _ok(_lib.wd_block_post(C.byref(dims), C.byref(w), _p(e0), _p(kv), batch, n_tok, _p(o), _p(X), _p(ws),
                           ws.numel() * ws.element_size(), _stream(stream)), "wd_block_post")


def wd_workspace_bytes_fp8(dims: wd_dims, batch: int) -> int:
    return _lib.wd_workspace_bytes_fp8(C.byref(dims), batch)


def wd_block_forward_fp8(dims, w: wd_block_weights, w8: wd_block_weights_fp8, e0, kv, batch, X, ws, stream=None):
    _ok(_lib.wd_block_forward_fp8(C.byref(dims), C.byref(w), C.byref(w8), _p(e0), _p(kv), batch, _p(X), _p(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "wd_block_forward_fp8")


def wd_unpatchify(dims, w: wd_head_weights, e, batch, X, v, ws, stream=None):
    _ok(_lib.wd_unpatchify(C.byref(dims), C.byref(w), _p(e), batch, _p(X), _p(v), _p(ws),
                           ws.numel() * ws.element_size(), _stream(stream)), "wd_unpatchify")


def wd_euler_cfg_step(x, v_cond, v_uncond, cfg_scale: float, dt: float, n=None, stream=None):
    n = x.numel() if n is None else n
    _ok(_lib.wd_euler_cfg_step(_p(x), _p(v_cond), _p(v_uncond), float(cfg_scale), float(dt), n, _stream(stream)),
        "wd_euler_cfg_step")


def wd_quant_rows_e4m3(dtype, rows, K, x, q, scale, stream=None):
    _ok(_lib.wd_quant_rows_e4m3(dtype, rows, K, _p(x), _p(q), _p(scale), _stream(stream)), "wd_quant_rows_e4m3")


def wd_gemm_fp8(M, N, K, Aq, sa, Bq, sb, bias, epilogue, out, gate_a=None, gate_b=None, stream=None):
    _ok(_lib.wd_gemm_fp8(M, N, K, _p(Aq), _p(sa), _p(Bq), _p(sb), _p(bias), epilogue, _p(out), _p(gate_a),
                         _p(gate_b), _stream(stream)), "wd_gemm_fp8")


def wd_gemm(dtype, M, N, K, A, B, bias, epilogue, out, gate_a=None, gate_b=None, stream=None):
    _ok(_lib.wd_gemm(dtype, M, N, K, _p(A), _p(B), _p(bias), epilogue, _p(out), _p(gate_a), _p(gate_b),
                     _stream(stream)), "wd_gemm")


def wd_attention(dtype, batch, Lq, heads, dh, q, k1, v1, n1, kv1_shared, o, k2=None, v2=None, n2=0, kv2_shared=0,
                 stream=None):
    _ok(_lib.wd_attention(dtype, batch, Lq, heads, dh, _p(q), _p(k1), _p(v1), n1, int(kv1_shared), _p(k2), _p(v2),
                          n2, int(kv2_shared), _p(o), _stream(stream)), "wd_attention")


def wd_test_exp2(x, y_fma, y_fma2, y_mufu, y_lib, stream=None):
    _ok(_lib.wd_test_exp2(_p(x), _p(y_fma), _p(y_fma2), _p(y_mufu), _p(y_lib), x.numel(), _stream(stream)),
        "wd_test_exp2")


def wd_test_gelu(x, y_as, y_as2, y_erf, stream=None):
    _ok(_lib.wd_test_gelu(_p(x), _p(y_as), _p(y_as2), _p(y_erf), x.numel(), _stream(stream)), "wd_test_gelu")


def wd_test_wait_timeout(limit_ns: int, site: int, out, stream=None):
    _ok(_lib.wd_test_wait_timeout(limit_ns, site, _p(out), _stream(stream)), "wd_test_wait_timeout")


def wd_check_status(stream=None) -> int:
    """wd_check's status code without raising (tests of the error path)."""
    return int(_lib.wd_check(_stream(stream)))


def wd_attention_lse(dtype, batch, Lq, heads, dh, q, k, v, n, kv_shared, o, lse, stream=None):
    _ok(_lib.wd_attention_lse(dtype, batch, Lq, heads, dh, _p(q), _p(k), _p(v), n, int(kv_shared), _p(o), _p(lse),
                              _stream(stream)), "wd_attention_lse")


def wd_attention_merge(dtype, batch, Lq, heads, dh, o_run, lse_run, o_part, lse_part, first, out=None, stream=None):
    _ok(_lib.wd_attention_merge(dtype, batch, Lq, heads, dh, _p(o_run), _p(lse_run), _p(o_part), _p(lse_part),
                                int(first), _p(out), _stream(stream)), "wd_attention_merge")


def wd_attention_fp8_layout(batch, Lq, Lk, heads, dh) -> wd_attn_fp8_layout:
    out = wd_attn_fp8_layout()
    _ok(_lib.wd_attention_fp8_layout(batch, Lq, Lk, heads, dh, C.byref(out)), "wd_attention_fp8_layout")
    return out


def wd_attention_fp8_quantize(batch, Lq, Lk, heads, dh, q, q_rs, k, v, kv_rs, buf, stream=None):
    _ok(_lib.wd_attention_fp8_quantize(batch, Lq, Lk, heads, dh, _p(q), q_rs, _p(k), _p(v), kv_rs, _p(buf),
                                       buf.numel() * buf.element_size(), _stream(stream)), "wd_attention_fp8_quantize")


def wd_attention_fp8(batch, Lq, Lk, heads, dh, buf, o, o_rs, stream=None):
    _ok(_lib.wd_attention_fp8(batch, Lq, Lk, heads, dh, _p(buf), buf.numel() * buf.element_size(), _p(o), o_rs,
                              _stream(stream)), "wd_attention_fp8")


def wd_set_debug_flags(flags: int):
    _lib.wd_set_debug_flags(flags)


def wd_debug_flags() -> int:
    return int(_lib.wd_debug_flags())


def wd_trace_enable(on: bool):
    _lib.wd_trace_enable(1 if on else 0)


def wd_trace_read():
    """{class: (launches, total device ms)} since the previous read."""
    n = (C.c_int64 * len(KERNEL_CLASSES))()
    ms = (C.c_double * len(KERNEL_CLASSES))()
    _ok(_lib.wd_trace_read(n, ms), "wd_trace_read")
    return {k: (int(n[i]), float(ms[i])) for i, k in enumerate(KERNEL_CLASSES)}
