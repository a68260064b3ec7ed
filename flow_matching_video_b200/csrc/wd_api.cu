// wd_api.cu — the extern "C" entry points of libwd: argument validation,
// workspace layout and the launch sequence of each step.
#include <cstdarg>
#include <cstring>

#include "wd_internal.cuh"

namespace wd {

static thread_local char g_msg[512] = "";
static unsigned g_debug_flags = 0;   // bit 0: SIMT GEMM for bf16, bit 1: SIMT attention for bf16

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

wd_status launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return WD_ERR_CUDA;
  }
  return WD_OK;
}

// ------------------------------------------------------------------ validation helpers
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define WD_NEED(p)                                                       \
  do {                                                                   \
    if ((p) == nullptr) { set_error("%s: %s is NULL", __func__, #p); return WD_ERR_ARG; } \
    if (!aligned16(p)) { set_error("%s: %s not 16-byte aligned", __func__, #p); return WD_ERR_ALIGN; } \
  } while (0)
#define WD_OPT(p)                                                        \
  do {                                                                   \
    if ((p) != nullptr && !aligned16(p)) { set_error("%s: %s not 16-byte aligned", __func__, #p); return WD_ERR_ALIGN; } \
  } while (0)

static wd_status check_dims(const wd_dims* d) {
  if (!d) { set_error("dims is NULL"); return WD_ERR_ARG; }
  if (d->dtype != WD_F32 && d->dtype != WD_BF16) { set_error("dims.dtype %d unknown", d->dtype); return WD_ERR_DTYPE; }
  if (d->norm != WD_NORM_LAYER && d->norm != WD_NORM_RMS) { set_error("dims.norm %d unknown", d->norm); return WD_ERR_ARG; }
  if (d->D <= 0 || d->heads <= 0 || d->D % d->heads) { set_error("D=%d heads=%d", d->D, d->heads); return WD_ERR_SHAPE; }
  const int dh = d->D / d->heads;
  if (dh != 32 && dh != 64 && dh != 128) { set_error("head dim %d unsupported (32, 64, 128)", dh); return WD_ERR_SHAPE; }
  if (d->D % 128) { set_error("D=%d must be a multiple of 128", d->D); return WD_ERR_SHAPE; }
  // The bf16 model runs its attention on the tensor cores, which take 128-wide heads only;
  // other widths would fall back to the CUDA-core kernel, so a model asking for them is refused.
  if (d->dtype == WD_BF16 && dh != 128) {
    set_error("bf16 model: head dim %d has no tensor-core attention (128 only)", dh);
    return WD_ERR_UNSUPPORTED;
  }
  if (d->ffn <= 0 || d->ffn % 64) { set_error("ffn=%d must be a positive multiple of 64", d->ffn); return WD_ERR_SHAPE; }
  if (d->T <= 0 || d->T > 256 || d->H <= 0 || d->W <= 0 || (d->H & 1) || (d->W & 1)) {
    set_error("latent grid T=%d H=%d W=%d (T<=256, H and W even)", d->T, d->H, d->W);
    return WD_ERR_SHAPE;
  }
  // n_img = 0 selects the text-to-video model (no image branch, c_img unused)
  if (d->n_txt <= 0 || d->n_img < 0 || d->c_txt <= 0 || (d->c_txt % 8) || (d->n_img > 0 && (d->c_img <= 0 || d->c_img % 8))) {
    set_error("context sizes n_txt=%d c_txt=%d n_img=%d c_img=%d", d->n_txt, d->c_txt, d->n_img, d->c_img);
    return WD_ERR_SHAPE;
  }
  if (!(d->eps > 0.f)) { set_error("eps must be > 0"); return WD_ERR_ARG; }
  return WD_OK;
}

static wd_status check_batch(int batch) {
  if (batch <= 0 || batch > 64) { set_error("batch=%d (1..64)", batch); return WD_ERR_SHAPE; }
  return WD_OK;
}

static int64_t tokens(const wd_dims* d) { return static_cast<int64_t>(d->T) * (d->H / 2) * (d->W / 2); }
static size_t esize(const wd_dims* d) { return d->dtype == WD_BF16 ? 2 : 4; }
// Patch width of the patch embedding: 36 input channels x (1,2,2) for the
// image-to-video model, 16 x (1,2,2) for the text-to-video model (n_img = 0).
static int patch_k(const wd_dims* d) { return d->n_img > 0 ? 144 : 64; }
static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout (each part 256-byte aligned):
//   bufA  [rows, max(3D, ffn)]  q|k|v, then qc, then the FFN hidden u
//   bufB  [rows, max(D, 144)]   h, patch gather, o, hc, oc, h2, head z
//   rope  [(T + H/2 + W/2), dh/2] float2 cos/sin table
struct Ws {
  void* a;
  void* b;
  float2* rope;
  size_t bytes;
};
static Ws ws_layout(const wd_dims* d, int batch, void* base) {
  const size_t rows = static_cast<size_t>(batch) * tokens(d);
  const size_t es = esize(d);
  const size_t wa = static_cast<size_t>(d->ffn > 3 * d->D ? d->ffn : 3 * d->D);
  const size_t wb = static_cast<size_t>(d->D > 144 ? d->D : 144);
  const size_t na = up256(rows * wa * es), nb = up256(rows * wb * es);
  const size_t nr = up256(static_cast<size_t>(d->T + d->H / 2 + d->W / 2) * (d->D / d->heads / 2) * sizeof(float2));
  char* p = static_cast<char*>(base);
  Ws w;
  w.a = p;
  w.b = p ? p + na : nullptr;
  w.rope = p ? reinterpret_cast<float2*>(p + na + nb) : nullptr;
  w.bytes = na + nb + nr;
  return w;
}

// ------------------------------------------------------------------ typed dispatch
template <typename T>
static wd_status gemm(int M, int N, int K, const void* A, int64_t lda, const void* B, int64_t ldb, int mode,
                      const Epi& ep, cudaStream_t st) {
  if constexpr (sizeof(T) == 2) {
    if (!(g_debug_flags & 1u))
      return gemm_tc(M, N, K, static_cast<const bf16*>(A), lda, static_cast<const bf16*>(B), ldb, mode, ep, st);
  }
  return gemm_simt<T>(M, N, K, static_cast<const T*>(A), lda, static_cast<const T*>(B), ldb, mode, ep, st);
}

template <typename TI, typename TO>
static wd_status attention(const AttnArgs<TI, TO>& a, cudaStream_t st) {
  if constexpr (sizeof(TI) == 2) {
    if (!(g_debug_flags & 2u) && a.dh == 128) return attention_tc(a, st);
  }
  return attention_simt<TI, TO>(a, st);
}

// Element type of the cross-attention operands (qc and the K/V cache): IEEE
// half on the bf16 path, where the text cross-attention's sharp softmax
// amplifies operand rounding; the activation type otherwise.
template <typename T> struct CrossT { using type = T; static constexpr int store = EPI_STORE; };
template <> struct CrossT<bf16> { using type = f16; static constexpr int store = EPI_STORE_F16; };

static Epi epi(void* out, int64_t ldo, const float* bias, const float* ga = nullptr, const float* gb = nullptr) {
  Epi e{};
  e.out = out; e.ldo = ldo; e.bias = bias; e.gate_a = ga; e.gate_b = gb;
  return e;
}

template <typename T>
static wd_status norm_rows(const wd_dims* d, const float* x, int64_t rows, const float* sh_a, const float* sh_b,
                           const float* sc_a, const float* sc_b, const float* g, const float* be, int rms, void* out,
                           cudaStream_t st) {
  NormArgs a{};
  a.x = x; a.rows = rows; a.D = d->D;
  a.sh_a = sh_a; a.sh_b = sh_b; a.sc_a = sc_a; a.sc_b = sc_b; a.gamma = g; a.beta = be;
  a.rms = rms; a.eps = d->eps; a.out = out;
  return norm_mod<T>(a, st);
}

// ------------------------------------------------------------------ block forward
// One block is three pieces, in this order, all on the same stream:
//   block_qkv_t        h = norm1(X)(1 + scale1) + shift1, q|k|v = h Wqkv^T + b,
//                      QK-RMSNorm + 3D RoPE in place (rows: a token slice)
//   self_attention_t   o = softmax(q k^T / sqrt(dh)) v over the whole sequence
//   block_post_t       X += gate1 (o Wo^T + b), the cross-attention, the FFN
//                      (rows: a token slice; every step here is row-local or
//                      reads only the context's keys and values)
// wd_block_forward runs them on the whole sequence with its workspace; the
// split entry points run them one by one (token slices for sequence
// parallelism, reused attention outputs for the attention cache).

template <typename T>
static wd_status block_qkv_t(const wd_dims* d, const wd_block_weights* w, const float* e0, int batch, int64_t tok0,
                             int64_t n_tok, const float* X, T* qkv, const Ws& ws, cudaStream_t st) {
  const int D = d->D, dh = D / d->heads;
  const int64_t rows = batch * n_tok;
  T* Bf = static_cast<T*>(ws.b);
  const float* mod = w->mod;
  // 1. h = norm(X)(1 + scale1) + shift1
  WD_TRY(norm_rows<T>(d, X, rows, e0, mod, e0 + D, mod + D, nullptr, nullptr, d->norm == WD_NORM_RMS, Bf, st));
  // 2. q|k|v = h Wqkv^T + b
  WD_TRY(gemm<T>(static_cast<int>(rows), 3 * D, D, Bf, D, w->qkv_w, D, EPI_STORE, epi(qkv, 3 * D, w->qkv_b), st));
  // 3. QK-RMSNorm + 3D RoPE in place (the cos/sin table lives in the workspace; it is
  //    rebuilt here because the library cannot assume the caller left it intact)
  { Trace tr(KC_SMALL, st); k_rope_table<<<64, 256, 0, st>>>(ws.rope, d->T, d->H / 2, d->W / 2, dh); }
  WD_TRY(launch_status("rope_table"));
  return qknorm_rope<T>(qkv, rows, *d, w->g_q, w->g_k, ws.rope, n_tok, tok0, st);
}

// Full self-attention over the fused projection buffer qkv [batch, L, 3 * heads * dh]
// (q of `heads` heads, then k, then v) -> o [batch, L, heads * dh].
template <typename T>
static wd_status self_attention_t(const wd_dims* d, int batch, int heads, const T* qkv, T* o, cudaStream_t st) {
  const int dh = d->D / d->heads, Dh = heads * dh;
  const int64_t L = tokens(d);
  AttnArgs<T, T> a{};
  a.q = qkv; a.q_rs = 3 * Dh;
  a.k1 = qkv + Dh; a.v1 = qkv + 2 * Dh; a.kv1_rs = 3 * Dh; a.kv1_bs = L * 3 * Dh; a.n1 = static_cast<int>(L);
  a.o = o; a.o_rs = Dh;
  a.batch = batch; a.Lq = static_cast<int>(L); a.heads = heads; a.dh = dh;
  return attention(a, st);
}

// The decoupled cross-attention ("图解 Wan2.1 I2V" 5.4) of n_tok queries per sample:
// qc [batch, n_tok, D] in the cross operand type, kv the block's K/V cache, oc [batch, n_tok, D].
template <typename T>
static wd_status cross_attention_t(const wd_dims* d, const void* kv, int batch, int64_t n_tok, const void* qc, T* oc,
                                   cudaStream_t st) {
  const int D = d->D, dh = D / d->heads;
  using CT = typename CrossT<T>::type;
  const size_t es = sizeof(CT);
  const char* kvp = static_cast<const char*>(kv);
  const size_t n_img_b = up256(static_cast<size_t>(d->n_img) * D * es);
  const size_t n_txt_b = up256(static_cast<size_t>(batch) * d->n_txt * D * es);
  const CT* k_img = reinterpret_cast<const CT*>(kvp);
  const CT* v_img = reinterpret_cast<const CT*>(kvp + n_img_b);
  const CT* k_txt = reinterpret_cast<const CT*>(kvp + 2 * n_img_b);
  const CT* v_txt = reinterpret_cast<const CT*>(kvp + 2 * n_img_b + n_txt_b);
  AttnArgs<CT, T> a{};
  a.q = static_cast<const CT*>(qc); a.q_rs = D;
  a.cross = true;
  if (d->n_img > 0) {
    a.k1 = k_img; a.v1 = v_img; a.kv1_rs = D; a.kv1_bs = 0; a.n1 = d->n_img;
    a.k2 = k_txt; a.v2 = v_txt; a.kv2_rs = D; a.kv2_bs = static_cast<int64_t>(d->n_txt) * D; a.n2 = d->n_txt;
  } else {   // text-to-video: one stream, text keys only ("图解 Wan2.1 I2V" 9)
    a.k1 = k_txt; a.v1 = v_txt; a.kv1_rs = D; a.kv1_bs = static_cast<int64_t>(d->n_txt) * D; a.n1 = d->n_txt;
  }
  a.o = oc; a.o_rs = D;
  a.batch = batch; a.Lq = static_cast<int>(n_tok); a.heads = d->heads; a.dh = dh;
  return attention(a, st);
}

template <typename T>
static wd_status block_post_t(const wd_dims* d, const wd_block_weights* w, const float* e0, const void* kv, int batch,
                              int64_t n_tok, const T* o, float* X, const Ws& ws, cudaStream_t st) {
  const int D = d->D, F = d->ffn, dh = D / d->heads;
  const int64_t rows = batch * n_tok;
  const int M = static_cast<int>(rows);
  T* A = static_cast<T*>(ws.a);
  T* Bf = static_cast<T*>(ws.b);
  const int rms = d->norm == WD_NORM_RMS;
  const float* mod = w->mod;

  // 5. X += gate1 * (o Wo^T + b)
  WD_TRY(gemm<T>(M, D, D, o, D, w->o_w, D, EPI_RESID, epi(X, D, w->o_b, e0 + 2 * D, mod + 2 * D), st));
  // 6. hc = LN_affine(X);  7. qc = hc Wcq^T + b
  WD_TRY(norm_rows<T>(d, X, rows, nullptr, nullptr, nullptr, nullptr, w->cn_g, w->cn_b, 0, Bf, st));
  WD_TRY(gemm<T>(M, D, D, Bf, D, w->cq_w, D, CrossT<T>::store, epi(A, D, w->cq_b), st));
  // 8. oc = attn(qc, K_img, V_img) + attn(qc, K_txt, V_txt)
  WD_TRY(cross_attention_t<T>(d, kv, batch, n_tok, A, Bf, st));
  // 9. X += oc Wco^T + b
  WD_TRY(gemm<T>(M, D, D, Bf, D, w->co_w, D, EPI_RESID, epi(X, D, w->co_b), st));
  // 10. h2 = norm(X)(1 + scale2) + shift2;  11. u = GELU(h2 W1^T + b1);  12. X += gate2 * (u W2^T + b2)
  WD_TRY(norm_rows<T>(d, X, rows, e0 + 3 * D, mod + 3 * D, e0 + 4 * D, mod + 4 * D, nullptr, nullptr, rms, Bf, st));
  WD_TRY(gemm<T>(M, F, D, Bf, D, w->f1_w, D, EPI_GELU, epi(A, F, w->f1_b), st));
  WD_TRY(gemm<T>(M, D, F, A, F, w->f2_w, F, EPI_RESID, epi(X, D, w->f2_b, e0 + 5 * D, mod + 5 * D), st));
  return WD_OK;
}

// ------------------------------------------------------------------ FP8 block
// The block of block_forward_t with its six linear layers on e4m3 operands
// ("Wan（通义万相）..." 5.3: FP8 GEMM, per-token activation scales; here per-output-
// channel weight scales): each GEMM input is quantised per row -- the three norms
// quantise their fp32 output in the same kernel, the attention outputs and the FFN
// hidden (bf16) go through the row quantiser -- and the GEMMs scale their fp32
// accumulators by both scales before the usual epilogues.  The attentions, the
// QK-norm + RoPE and the residual stream are those of the bf16 block.
// Workspace: the bf16 block's, then the e4m3 activations [rows, max(D, ffn)] and
// their row scales [rows].
struct Ws8 {
  Ws base;
  uint8_t* q;
  float* s;
  void* attn8;                 // the FP8 attention's operands (layout a8)
  wd_attn_fp8_layout a8;
  size_t bytes;
};
static Ws8 ws_layout_fp8(const wd_dims* d, int batch, void* base) {
  Ws8 w;
  w.base = ws_layout(d, batch, base);
  const size_t rows = static_cast<size_t>(batch) * tokens(d);
  const size_t nq = up256(rows * static_cast<size_t>(d->ffn > d->D ? d->ffn : d->D));
  const size_t ns = up256(rows * sizeof(float));
  w.a8 = wd_attn_fp8_layout{};
  const int dh = d->D / d->heads;
  if (dh != 128 || attn_fp8_layout(batch, tokens(d), tokens(d), d->heads, dh, &w.a8) != WD_OK) w.a8.bytes = 0;
  char* p = base ? static_cast<char*>(base) + w.base.bytes : nullptr;
  w.q = reinterpret_cast<uint8_t*>(p);
  w.s = p ? reinterpret_cast<float*>(p + nq) : nullptr;
  w.attn8 = p ? p + nq + ns : nullptr;
  w.bytes = w.base.bytes + nq + ns + w.a8.bytes;
  return w;
}

static wd_status block_forward_fp8_t(const wd_dims* d, const wd_block_weights* w, const wd_block_weights_fp8* w8,
                                     const float* e0, const void* kv, int batch, float* X, const Ws8& ws,
                                     cudaStream_t st) {
  const int D = d->D, F = d->ffn, dh = D / d->heads;
  const int64_t L = tokens(d), rows = batch * L;
  const int M = static_cast<int>(rows);
  bf16* A = static_cast<bf16*>(ws.base.a);
  bf16* Bf = static_cast<bf16*>(ws.base.b);
  uint8_t* Q = ws.q;
  float* S = ws.s;
  const int rms = d->norm == WD_NORM_RMS;
  const float* mod = w->mod;
  // e4m3 GEMM on the quantised activations Q (row scales S) and a quantised weight
  auto g8 = [&](int N, int K, const void* wq, const float* wsc, const float* bias, int mode, void* out, int64_t ldo,
                const float* ga, const float* gb) -> wd_status {
    Epi ep = epi(out, ldo, bias, ga, gb);
    ep.sa = S;
    ep.sb = wsc;
    return gemm_tc_fp8(M, N, K, Q, K, static_cast<const uint8_t*>(wq), K, mode, ep, st);
  };
  // norm (+ modulate or affine) with its output quantised into Q, S
  auto nq = [&](const float* sh_a, const float* sh_b, const float* sc_a, const float* sc_b, const float* g,
                const float* be, int rms_) -> wd_status {
    NormArgs a{};
    a.x = X; a.rows = rows; a.D = D;
    a.sh_a = sh_a; a.sh_b = sh_b; a.sc_a = sc_a; a.sc_b = sc_b; a.gamma = g; a.beta = be;
    a.rms = rms_; a.eps = d->eps; a.out = Q; a.scale = S;
    return norm_mod<uint8_t>(a, st);
  };
  // 1. h = norm(X)(1 + scale1) + shift1, quantised;  2. q|k|v = h Wqkv^T + b
  WD_TRY(nq(e0, mod, e0 + D, mod + D, nullptr, nullptr, rms));
  WD_TRY(g8(3 * D, D, w8->qkv_q, w8->qkv_s, w->qkv_b, EPI_STORE, A, 3 * D, nullptr, nullptr));
  // 3. QK-RMSNorm + 3D RoPE;  4. self-attention -> o (bf16)
  { Trace tr(KC_SMALL, st); k_rope_table<<<64, 256, 0, st>>>(ws.base.rope, d->T, d->H / 2, d->W / 2, dh); }
  WD_TRY(launch_status("rope_table"));
  WD_TRY(qknorm_rope<bf16>(A, rows, *d, w->g_q, w->g_k, ws.base.rope, L, 0, st));
  if (w8->attention_fp8) {   // INT8 Q K^T, FP8 P V
    WD_TRY(attn_fp8_quantize(batch, static_cast<int>(L), static_cast<int>(L), d->heads, A, 3 * D, A + D, A + 2 * D,
                             3 * D, ws.attn8, ws.a8, st));
    WD_TRY(attn_fp8(batch, static_cast<int>(L), static_cast<int>(L), d->heads, ws.attn8, ws.a8, Bf, D, st));
  } else {
    WD_TRY(self_attention_t<bf16>(d, batch, d->heads, A, Bf, st));
  }
  // 5. X += gate1 * (o Wo^T + b), o quantised
  WD_TRY(quant_rows_e4m3<bf16>(M, D, Bf, Q, S, st));
  WD_TRY(g8(D, D, w8->o_q, w8->o_s, w->o_b, EPI_RESID, X, D, e0 + 2 * D, mod + 2 * D));
  // 6. hc = LN_affine(X), quantised;  7. qc = hc Wcq^T + b (IEEE half)
  WD_TRY(nq(nullptr, nullptr, nullptr, nullptr, w->cn_g, w->cn_b, 0));
  WD_TRY(g8(D, D, w8->cq_q, w8->cq_s, w->cq_b, EPI_STORE_F16, A, D, nullptr, nullptr));
  // 8. decoupled cross-attention -> oc (bf16);  9. X += oc Wco^T + b, oc quantised
  WD_TRY(cross_attention_t<bf16>(d, kv, batch, L, A, Bf, st));
  WD_TRY(quant_rows_e4m3<bf16>(M, D, Bf, Q, S, st));
  WD_TRY(g8(D, D, w8->co_q, w8->co_s, w->co_b, EPI_RESID, X, D, nullptr, nullptr));
  // 10. h2 = norm(X)(1 + scale2) + shift2, quantised;  11. u = GELU(h2 W1^T + b1) (bf16)
  WD_TRY(nq(e0 + 3 * D, mod + 3 * D, e0 + 4 * D, mod + 4 * D, nullptr, nullptr, rms));
  WD_TRY(g8(F, D, w8->f1_q, w8->f1_s, w->f1_b, EPI_GELU, A, F, nullptr, nullptr));
  // 12. X += gate2 * (u W2^T + b2): u quantised, or (no e4m3 FFN2 weight) the bf16 GEMM on u
  if (!w8->f2_q)
    return gemm<bf16>(M, D, F, A, F, w->f2_w, F, EPI_RESID, epi(X, D, w->f2_b, e0 + 5 * D, mod + 5 * D), st);
  WD_TRY(quant_rows_e4m3<bf16>(M, F, A, Q, S, st));
  return g8(D, F, w8->f2_q, w8->f2_s, w->f2_b, EPI_RESID, X, D, e0 + 5 * D, mod + 5 * D);
}

template <typename T>
static wd_status block_forward_t(const wd_dims* d, const wd_block_weights* w, const float* e0, const void* kv,
                                 int batch, float* X, const Ws& ws, cudaStream_t st) {
  const int64_t L = tokens(d);
  T* A = static_cast<T*>(ws.a);
  T* Bf = static_cast<T*>(ws.b);
  WD_TRY(block_qkv_t<T>(d, w, e0, batch, 0, L, X, A, ws, st));          // q|k|v -> bufA
  WD_TRY(self_attention_t<T>(d, batch, d->heads, A, Bf, st));           // o -> bufB
  return block_post_t<T>(d, w, e0, kv, batch, L, Bf, X, ws, st);
}

}  // namespace wd

using namespace wd;

// ====================================================================== C ABI
extern "C" {

const char* wd_last_error(void) { return g_msg; }
const char* wd_version(void) { return "libwd 0.1 sm_100a"; }

void wd_set_debug_flags(unsigned flags) { g_debug_flags = flags; }
unsigned wd_debug_flags(void) { return g_debug_flags; }

wd_status wd_check(wd_stream stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) { set_error("async CUDA error: %s", cudaGetErrorString(e)); return WD_ERR_CUDA; }
  unsigned err = 0;
  e = cudaMemcpyFromSymbol(&err, g_wd_error, sizeof(err));
  if (e != cudaSuccess) { set_error("reading device error word: %s", cudaGetErrorString(e)); return WD_ERR_CUDA; }
  if (err) {
    const unsigned zero = 0;
    cudaMemcpyToSymbol(g_wd_error, &zero, sizeof(zero));
    set_error("device wait ran out (site 0x%x)", err);
    return WD_ERR_TIMEOUT;
  }
  return WD_OK;
}

int64_t wd_token_count(const wd_dims* d) {
  if (!d || d->T <= 0 || d->H <= 0 || d->W <= 0) return 0;
  return tokens(d);
}

size_t wd_workspace_bytes(const wd_dims* d, int batch) {
  if (check_dims(d) != WD_OK || check_batch(batch) != WD_OK) return 0;
  return ws_layout(d, batch, nullptr).bytes;
}

size_t wd_ctx_bytes(const wd_dims* d, int batch) {
  if (check_dims(d) != WD_OK || check_batch(batch) != WD_OK) return 0;
  const size_t es = esize(d);
  const size_t hid = static_cast<size_t>(batch * d->n_txt > d->n_img ? batch * d->n_txt : d->n_img);
  return up256(static_cast<size_t>(batch) * d->n_txt * d->D * es) + up256(static_cast<size_t>(d->n_img) * d->D * es) +
         up256(hid * d->D * es);
}

size_t wd_kv_bytes(const wd_dims* d, int batch) {
  if (check_dims(d) != WD_OK || check_batch(batch) != WD_OK) return 0;
  const size_t es = esize(d);
  return 2 * up256(static_cast<size_t>(d->n_img) * d->D * es) +
         2 * up256(static_cast<size_t>(batch) * d->n_txt * d->D * es);
}

wd_status wd_build_cond_y(const wd_dims* d, const float* img_lat, const int* known_frames, int n_known, float* y,
                          wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_NEED(img_lat);
  WD_NEED(y);
  const int F = 4 * (d->T - 1) + 1;
  // pixel-frame sequence: frame 0 four times, then frames 1..F-1; latent frame f
  // channel c takes entry 4f + c ("图解 Wan2.1 I2V" 4.1 step 3).
  MaskBits mb{};
  int def = 0;
  const int* kf = (known_frames && n_known > 0) ? known_frames : &def;
  const int nk = (known_frames && n_known > 0) ? n_known : 1;
  for (int i = 0; i < nk; ++i) {
    const int p = kf[i];
    if (p < 0 || p >= F) { set_error("known frame %d outside [0, %d)", p, F); return WD_ERR_ARG; }
    if (p == 0) {
      for (int c = 0; c < 4; ++c) mb.w[c >> 5] |= 1u << (c & 31);
    } else {
      const int e = p + 3;
      mb.w[e >> 5] |= 1u << (e & 31);
    }
  }
  const int64_t HW = static_cast<int64_t>(d->H) * d->W;
  const int64_t n = 20 * d->T * HW;
  const unsigned grid = static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  Trace tr(KC_SMALL, static_cast<cudaStream_t>(stream));
  k_cond_y<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(img_lat, mb, d->T, HW, y);
  return launch_status("build_cond_y");
}

wd_status wd_euler_cfg_step(float* x, const float* v_cond, const float* v_uncond, float cfg_scale, float dt, size_t n,
                            wd_stream stream) {
  WD_NEED(x);
  WD_NEED(v_cond);
  WD_OPT(v_uncond);
  if (n == 0) return WD_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t want = (n / 4 + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < static_cast<size_t>(sms) * 8 ? (want ? want : 1) : sms * 8);
  Trace tr(KC_EULER, static_cast<cudaStream_t>(stream));
  k_euler_cfg<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, v_cond, v_uncond, cfg_scale, dt,
                                                                   static_cast<int64_t>(n));
  return launch_status("euler_cfg_step");
}

wd_status wd_time_mod(const wd_dims* d, const wd_time_weights* w, float tau, float* e, float* e0, wd_stream stream) {
  WD_TRY(check_dims(d));
  if (!w) { set_error("time weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->t1_w); WD_NEED(w->t1_b); WD_NEED(w->t2_w); WD_NEED(w->t2_b); WD_NEED(w->tp_w); WD_NEED(w->tp_b);
  WD_NEED(e);
  WD_NEED(e0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = d->D;
  // h1 = t1(sin(tau)) is written to e0 (scratch until the last launch)
  { Trace tr(KC_SMALL, st); k_time_matvec<<<(D * 32 + 255) / 256, 256, 0, st>>>(w->t1_w, w->t1_b, nullptr, tau, 0, D, 256, e0); }
  { Trace tr(KC_SMALL, st); k_time_matvec<<<(D * 32 + 255) / 256, 256, 0, st>>>(w->t2_w, w->t2_b, e0, 0.f, 1, D, D, e); }
  { Trace tr(KC_SMALL, st); k_time_matvec<<<(6 * D * 32 + 255) / 256, 256, 0, st>>>(w->tp_w, w->tp_b, e, 0.f, 1, 6 * D, D, e0); }
  return launch_status("time_mod");
}

wd_status wd_context_embed(const wd_dims* d, const wd_ctx_weights* w, const void* txt, const void* clip, int batch,
                           void* ctx, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  if (!w) { set_error("ctx weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->txt1_w); WD_NEED(w->txt1_b); WD_NEED(w->txt2_w); WD_NEED(w->txt2_b);
  const bool img = d->n_img > 0;   // the text-to-video model has no CLIP branch
  if (img) { WD_NEED(w->img1_w); WD_NEED(w->img1_b); WD_NEED(w->img2_w); WD_NEED(w->img2_b); WD_NEED(clip); }
  WD_NEED(txt);
  WD_NEED(ctx);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = d->D;
  const size_t es = esize(d);
  char* p = static_cast<char*>(ctx);
  void* ctx_txt = p;
  void* ctx_img = p + up256(static_cast<size_t>(batch) * d->n_txt * D * es);
  void* hid = static_cast<char*>(ctx_img) + up256(static_cast<size_t>(d->n_img) * D * es);
  const int Mt = batch * d->n_txt;
  if (d->dtype == WD_BF16) {
    WD_TRY(gemm<bf16>(Mt, D, d->c_txt, txt, d->c_txt, w->txt1_w, d->c_txt, EPI_GELU, epi(hid, D, w->txt1_b), st));
    WD_TRY(gemm<bf16>(Mt, D, D, hid, D, w->txt2_w, D, EPI_STORE, epi(ctx_txt, D, w->txt2_b), st));
    if (img) {
      WD_TRY(gemm<bf16>(d->n_img, D, d->c_img, clip, d->c_img, w->img1_w, d->c_img, EPI_GELU, epi(hid, D, w->img1_b), st));
      WD_TRY(gemm<bf16>(d->n_img, D, D, hid, D, w->img2_w, D, EPI_STORE, epi(ctx_img, D, w->img2_b), st));
    }
  } else {
    WD_TRY(gemm<float>(Mt, D, d->c_txt, txt, d->c_txt, w->txt1_w, d->c_txt, EPI_GELU, epi(hid, D, w->txt1_b), st));
    WD_TRY(gemm<float>(Mt, D, D, hid, D, w->txt2_w, D, EPI_STORE, epi(ctx_txt, D, w->txt2_b), st));
    if (img) {
      WD_TRY(gemm<float>(d->n_img, D, d->c_img, clip, d->c_img, w->img1_w, d->c_img, EPI_GELU, epi(hid, D, w->img1_b), st));
      WD_TRY(gemm<float>(d->n_img, D, D, hid, D, w->img2_w, D, EPI_STORE, epi(ctx_img, D, w->img2_b), st));
    }
  }
  return WD_OK;
}

wd_status wd_cross_kv(const wd_dims* d, const wd_block_weights* w, const void* ctx, int batch, void* kv,
                      wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  if (!w) { set_error("block weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->ck_w); WD_NEED(w->ck_b); WD_NEED(w->cv_w); WD_NEED(w->cv_b);
  const bool img = d->n_img > 0;   // the text-to-video model has text keys and values only
  if (img) { WD_NEED(w->cki_w); WD_NEED(w->cki_b); WD_NEED(w->cvi_w); WD_NEED(w->cvi_b); }
  WD_NEED(ctx);
  WD_NEED(kv);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = d->D;
  const size_t es = esize(d);   // context and K/V cache elements: 2 bytes (bf16 / IEEE half) or 4 (fp32)
  const char* p = static_cast<const char*>(ctx);
  const void* ctx_txt = p;
  const void* ctx_img = p + up256(static_cast<size_t>(batch) * d->n_txt * D * es);
  char* q = static_cast<char*>(kv);
  const size_t ni = up256(static_cast<size_t>(d->n_img) * D * es), nt = up256(static_cast<size_t>(batch) * d->n_txt * D * es);
  void *k_img = q, *v_img = q + ni, *k_txt = q + 2 * ni, *v_txt = q + 2 * ni + nt;
  const int Mt = batch * d->n_txt;
  if (d->dtype == WD_BF16) {
    // stored as IEEE half: the cross-attention operands of the bf16 path
    if (img) {
      WD_TRY(gemm<bf16>(d->n_img, D, D, ctx_img, D, w->cki_w, D, EPI_STORE_F16, epi(k_img, D, w->cki_b), st));
      WD_TRY(gemm<bf16>(d->n_img, D, D, ctx_img, D, w->cvi_w, D, EPI_STORE_F16, epi(v_img, D, w->cvi_b), st));
    }
    WD_TRY(gemm<bf16>(Mt, D, D, ctx_txt, D, w->ck_w, D, EPI_STORE_F16, epi(k_txt, D, w->ck_b), st));
    WD_TRY(gemm<bf16>(Mt, D, D, ctx_txt, D, w->cv_w, D, EPI_STORE_F16, epi(v_txt, D, w->cv_b), st));
  } else {
    if (img) {
      WD_TRY(gemm<float>(d->n_img, D, D, ctx_img, D, w->cki_w, D, EPI_STORE, epi(k_img, D, w->cki_b), st));
      WD_TRY(gemm<float>(d->n_img, D, D, ctx_img, D, w->cvi_w, D, EPI_STORE, epi(v_img, D, w->cvi_b), st));
    }
    WD_TRY(gemm<float>(Mt, D, D, ctx_txt, D, w->ck_w, D, EPI_STORE, epi(k_txt, D, w->ck_b), st));
    WD_TRY(gemm<float>(Mt, D, D, ctx_txt, D, w->cv_w, D, EPI_STORE, epi(v_txt, D, w->cv_b), st));
  }
  return WD_OK;
}

wd_status wd_patch_embed(const wd_dims* d, const float* x_t, const float* y, const void* w, const float* b, int batch,
                         float* X, void* ws, size_t ws_bytes, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  WD_NEED(x_t); WD_NEED(w); WD_NEED(b); WD_NEED(X); WD_NEED(ws);
  if (d->n_img > 0) { WD_NEED(y); } else { WD_OPT(y); }
  const Ws L = ws_layout(d, batch, ws);
  if (ws_bytes < L.bytes) { set_error("workspace %zu < %zu bytes", ws_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = batch * tokens(d);
  const int K = patch_k(d);
  const int64_t n = rows * K;
  const unsigned grid = static_cast<unsigned>((n + 255) / 256 < 65536 ? (n + 255) / 256 : 65536);
  if (d->dtype == WD_BF16) {
    { Trace tr(KC_SMALL, st); k_patch_gather<bf16><<<grid, 256, 0, st>>>(x_t, y, batch, d->T, d->H, d->W, K, static_cast<bf16*>(L.b)); }
    WD_TRY(launch_status("patch_gather"));
    WD_TRY(gemm<bf16>(static_cast<int>(rows), d->D, K, L.b, K, w, K, EPI_F32, epi(X, d->D, b), st));
  } else {
    { Trace tr(KC_SMALL, st); k_patch_gather<float><<<grid, 256, 0, st>>>(x_t, y, batch, d->T, d->H, d->W, K, static_cast<float*>(L.b)); }
    WD_TRY(launch_status("patch_gather"));
    WD_TRY(gemm<float>(static_cast<int>(rows), d->D, K, L.b, K, w, K, EPI_F32, epi(X, d->D, b), st));
  }
  return WD_OK;
}

wd_status wd_block_forward(const wd_dims* d, const wd_block_weights* w, const float* e0, const void* kv, int batch,
                           float* X, void* ws, size_t ws_bytes, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  if (!w) { set_error("block weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->qkv_w); WD_NEED(w->qkv_b); WD_NEED(w->g_q); WD_NEED(w->g_k); WD_NEED(w->o_w); WD_NEED(w->o_b);
  WD_NEED(w->cn_g); WD_NEED(w->cn_b); WD_NEED(w->cq_w); WD_NEED(w->cq_b); WD_NEED(w->co_w); WD_NEED(w->co_b);
  WD_NEED(w->f1_w); WD_NEED(w->f1_b); WD_NEED(w->f2_w); WD_NEED(w->f2_b); WD_NEED(w->mod);
  WD_NEED(e0); WD_NEED(kv); WD_NEED(X); WD_NEED(ws);
  const Ws L = ws_layout(d, batch, ws);
  if (ws_bytes < L.bytes) { set_error("workspace %zu < %zu bytes", ws_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  if (static_cast<int64_t>(batch) * tokens(d) > 0x7fffffff) { set_error("too many rows"); return WD_ERR_SHAPE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == WD_BF16) return block_forward_t<bf16>(d, w, e0, kv, batch, X, L, st);
  return block_forward_t<float>(d, w, e0, kv, batch, X, L, st);
}

// The three pieces of wd_block_forward, callable one by one.
static wd_status check_slice(const wd_dims* d, int64_t tok0, int64_t n_tok) {
  const int64_t L = tokens(d);
  if (n_tok <= 0 || tok0 < 0 || tok0 + n_tok > L) {
    set_error("token slice [%lld, %lld) outside the sequence [0, %lld)", (long long)tok0, (long long)(tok0 + n_tok),
              (long long)L);
    return WD_ERR_SHAPE;
  }
  return WD_OK;
}

wd_status wd_block_qkv(const wd_dims* d, const wd_block_weights* w, const float* e0, int batch, int64_t tok0,
                       int64_t n_tok, const float* X, void* qkv, void* ws, size_t ws_bytes, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  WD_TRY(check_slice(d, tok0, n_tok));
  if (!w) { set_error("block weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->qkv_w); WD_NEED(w->qkv_b); WD_NEED(w->g_q); WD_NEED(w->g_k); WD_NEED(w->mod);
  WD_NEED(e0); WD_NEED(X); WD_NEED(qkv); WD_NEED(ws);
  const Ws L = ws_layout(d, batch, ws);
  if (ws_bytes < L.bytes) { set_error("workspace %zu < %zu bytes", ws_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == WD_BF16) return block_qkv_t<bf16>(d, w, e0, batch, tok0, n_tok, X, static_cast<bf16*>(qkv), L, st);
  return block_qkv_t<float>(d, w, e0, batch, tok0, n_tok, X, static_cast<float*>(qkv), L, st);
}

wd_status wd_block_self_attention(const wd_dims* d, int batch, int heads, const void* qkv, void* o, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  if (heads <= 0 || heads > d->heads) { set_error("heads=%d (1..%d)", heads, d->heads); return WD_ERR_SHAPE; }
  WD_NEED(qkv); WD_NEED(o);
  if (batch * tokens(d) > 0x7fffffff) { set_error("too many rows"); return WD_ERR_SHAPE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == WD_BF16)
    return self_attention_t<bf16>(d, batch, heads, static_cast<const bf16*>(qkv), static_cast<bf16*>(o), st);
  return self_attention_t<float>(d, batch, heads, static_cast<const float*>(qkv), static_cast<float*>(o), st);
}

wd_status wd_block_post(const wd_dims* d, const wd_block_weights* w, const float* e0, const void* kv, int batch,
                        int64_t n_tok, const void* o, float* X, void* ws, size_t ws_bytes, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  WD_TRY(check_slice(d, 0, n_tok));
  if (!w) { set_error("block weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->o_w); WD_NEED(w->o_b); WD_NEED(w->cn_g); WD_NEED(w->cn_b); WD_NEED(w->cq_w); WD_NEED(w->cq_b);
  WD_NEED(w->co_w); WD_NEED(w->co_b); WD_NEED(w->f1_w); WD_NEED(w->f1_b); WD_NEED(w->f2_w); WD_NEED(w->f2_b);
  WD_NEED(w->mod);
  WD_NEED(e0); WD_NEED(kv); WD_NEED(o); WD_NEED(X); WD_NEED(ws);
  const Ws L = ws_layout(d, batch, ws);
  if (ws_bytes < L.bytes) { set_error("workspace %zu < %zu bytes", ws_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->dtype == WD_BF16) return block_post_t<bf16>(d, w, e0, kv, batch, n_tok, static_cast<const bf16*>(o), X, L, st);
  return block_post_t<float>(d, w, e0, kv, batch, n_tok, static_cast<const float*>(o), X, L, st);
}

size_t wd_workspace_bytes_fp8(const wd_dims* d, int batch) {
  if (check_dims(d) != WD_OK || check_batch(batch) != WD_OK) return 0;
  return ws_layout_fp8(d, batch, nullptr).bytes;
}

wd_status wd_block_forward_fp8(const wd_dims* d, const wd_block_weights* w, const wd_block_weights_fp8* w8,
                               const float* e0, const void* kv, int batch, float* X, void* ws, size_t ws_bytes,
                               wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  if (d->dtype != WD_BF16) { set_error("wd_block_forward_fp8: the FP8 block is the bf16 model's"); return WD_ERR_UNSUPPORTED; }
  if (d->D % 256 || d->ffn % 256) {
    set_error("wd_block_forward_fp8: D=%d and ffn=%d must be multiples of 256", d->D, d->ffn);
    return WD_ERR_SHAPE;
  }
  if (!w || !w8) { set_error("block weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->qkv_b); WD_NEED(w->g_q); WD_NEED(w->g_k); WD_NEED(w->o_b); WD_NEED(w->cn_g); WD_NEED(w->cn_b);
  WD_NEED(w->cq_b); WD_NEED(w->co_b); WD_NEED(w->f1_b); WD_NEED(w->f2_b); WD_NEED(w->mod);
  WD_NEED(w8->qkv_q); WD_NEED(w8->o_q); WD_NEED(w8->cq_q); WD_NEED(w8->co_q); WD_NEED(w8->f1_q);
  WD_NEED(w8->qkv_s); WD_NEED(w8->o_s); WD_NEED(w8->cq_s); WD_NEED(w8->co_s); WD_NEED(w8->f1_s);
  if (w8->f2_q) { WD_NEED(w8->f2_s); } else { WD_NEED(w->f2_w); }   // no e4m3 FFN2: the bf16 weight
  if (w8->attention_fp8 && d->D / d->heads != 128) {
    set_error("wd_block_forward_fp8: the FP8 attention needs 128-wide heads");
    return WD_ERR_UNSUPPORTED;
  }
  WD_NEED(e0); WD_NEED(kv); WD_NEED(X); WD_NEED(ws);
  const Ws8 L = ws_layout_fp8(d, batch, ws);
  if (ws_bytes < L.bytes) { set_error("workspace %zu < %zu bytes", ws_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  if (static_cast<int64_t>(batch) * tokens(d) > 0x7fffffff) { set_error("too many rows"); return WD_ERR_SHAPE; }
  return block_forward_fp8_t(d, w, w8, e0, kv, batch, X, L, static_cast<cudaStream_t>(stream));
}

wd_status wd_unpatchify(const wd_dims* d, const wd_head_weights* w, const float* e, int batch, const float* X, float* v,
                        void* ws, size_t ws_bytes, wd_stream stream) {
  WD_TRY(check_dims(d));
  WD_TRY(check_batch(batch));
  if (!w) { set_error("head weights NULL"); return WD_ERR_ARG; }
  WD_NEED(w->mod); WD_NEED(w->w); WD_NEED(w->b);
  WD_NEED(e); WD_NEED(X); WD_NEED(v); WD_NEED(ws);
  const Ws L = ws_layout(d, batch, ws);
  if (ws_bytes < L.bytes) { set_error("workspace %zu < %zu bytes", ws_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int D = d->D;
  const int64_t rows = batch * tokens(d);
  Epi ep = epi(v, 0, w->b);
  ep.T = d->T; ep.Hp = d->H / 2; ep.Wp = d->W / 2; ep.L = static_cast<int>(tokens(d));
  if (d->dtype == WD_BF16) {
    WD_TRY(norm_rows<bf16>(d, X, rows, e, w->mod, e, w->mod + D, nullptr, nullptr, 0, L.b, st));
    WD_TRY(gemm<bf16>(static_cast<int>(rows), 64, D, L.b, D, w->w, D, EPI_UNPATCH, ep, st));
  } else {
    WD_TRY(norm_rows<float>(d, X, rows, e, w->mod, e, w->mod + D, nullptr, nullptr, 0, L.b, st));
    WD_TRY(gemm<float>(static_cast<int>(rows), 64, D, L.b, D, w->w, D, EPI_UNPATCH, ep, st));
  }
  return WD_OK;
}

// ---------------------------------------------------------------- building blocks (tested one by one)
// C = epilogue(A[M,K] B[N,K]^T) with the epilogue codes of the block
// (0 store, 1 GELU, 2 fp32 store, 3 gated residual add into fp32 out,
// 5 IEEE half store, bf16 inputs only).
wd_status wd_gemm(int dtype, int M, int N, int K, const void* A, const void* B, const float* bias, int epilogue,
                  void* out, const float* gate_a, const float* gate_b, wd_stream stream) {
  WD_NEED(A); WD_NEED(B); WD_NEED(out); WD_OPT(bias); WD_OPT(gate_a); WD_OPT(gate_b);
  if (epilogue < 0 || epilogue > 5 || epilogue == EPI_UNPATCH || (epilogue == EPI_STORE_F16 && dtype != WD_BF16)) {
    set_error("epilogue %d (dtype %d)", epilogue, dtype);
    return WD_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Epi ep = epi(out, N, bias, gate_a, gate_b);
  if (dtype == WD_BF16) return gemm<bf16>(M, N, K, A, K, B, K, epilogue, ep, st);
  if (dtype == WD_F32) return gemm<float>(M, N, K, A, K, B, K, epilogue, ep, st);
  set_error("dtype %d", dtype);
  return WD_ERR_DTYPE;
}

// Per-row e4m3 quantisation and the FP8 GEMM ("Wan（通义万相）..." 5.3).
wd_status wd_quant_rows_e4m3(int dtype, int rows, int K, const void* x, void* q, float* scale, wd_stream stream) {
  WD_NEED(x); WD_NEED(q); WD_NEED(scale);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == WD_BF16) return quant_rows_e4m3<bf16>(rows, K, static_cast<const bf16*>(x), static_cast<uint8_t*>(q), scale, st);
  if (dtype == WD_F32) return quant_rows_e4m3<float>(rows, K, static_cast<const float*>(x), static_cast<uint8_t*>(q), scale, st);
  set_error("dtype %d", dtype);
  return WD_ERR_DTYPE;
}

wd_status wd_gemm_fp8(int M, int N, int K, const void* Aq, const float* sa, const void* Bq, const float* sb,
                      const float* bias, int epilogue, void* out, const float* gate_a, const float* gate_b,
                      wd_stream stream) {
  WD_NEED(Aq); WD_NEED(sa); WD_NEED(Bq); WD_NEED(sb); WD_NEED(out); WD_OPT(bias); WD_OPT(gate_a); WD_OPT(gate_b);
  if (epilogue < 0 || (epilogue > EPI_RESID && epilogue != EPI_STORE_F16)) {
    set_error("gemm_fp8: epilogue %d (0-3, 5)", epilogue);
    return WD_ERR_ARG;
  }
  Epi ep = epi(out, N, bias, gate_a, gate_b);
  ep.sa = sa;
  ep.sb = sb;
  return gemm_tc_fp8(M, N, K, static_cast<const uint8_t*>(Aq), K, static_cast<const uint8_t*>(Bq), K, epilogue, ep,
                     static_cast<cudaStream_t>(stream));
}

// O[b, l, h*dh:(h+1)*dh] = softmax(q k^T / sqrt(dh)) v  (+ second segment).
// q [batch, Lq, heads*dh]; k1/v1 [batch or 1 (kv1_shared), n1, heads*dh];
// k2/v2 likewise or NULL; o [batch, Lq, heads*dh] (bf16 when the operands
// are IEEE half).
wd_status wd_attention(int dtype, int batch, int Lq, int heads, int dh, const void* q, const void* k1, const void* v1,
                       int n1, int kv1_shared, const void* k2, const void* v2, int n2, int kv2_shared, void* o,
                       wd_stream stream) {
  WD_NEED(q); WD_NEED(k1); WD_NEED(v1); WD_NEED(o); WD_OPT(k2); WD_OPT(v2);
  if (batch <= 0 || Lq <= 0 || heads <= 0 || n1 <= 0 || (k2 && n2 <= 0)) { set_error("attention sizes"); return WD_ERR_SHAPE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t D = static_cast<int64_t>(heads) * dh;
  auto fill = [&](auto a) {
    a.cross = k2 != nullptr;
    a.q_rs = D; a.kv1_rs = D; a.kv1_bs = kv1_shared ? 0 : n1 * D; a.n1 = n1;
    a.kv2_rs = D; a.kv2_bs = kv2_shared ? 0 : n2 * D; a.n2 = k2 ? n2 : 0;
    a.o_rs = D; a.batch = batch; a.Lq = Lq; a.heads = heads; a.dh = dh;
    return a;
  };
  if (dtype == WD_BF16) {
    AttnArgs<bf16, bf16> a{};
    a.q = static_cast<const bf16*>(q); a.k1 = static_cast<const bf16*>(k1); a.v1 = static_cast<const bf16*>(v1);
    a.k2 = static_cast<const bf16*>(k2); a.v2 = static_cast<const bf16*>(v2); a.o = static_cast<bf16*>(o);
    return attention(fill(a), st);
  }
  if (dtype == WD_F16) {
    AttnArgs<f16, bf16> a{};
    a.q = static_cast<const f16*>(q); a.k1 = static_cast<const f16*>(k1); a.v1 = static_cast<const f16*>(v1);
    a.k2 = static_cast<const f16*>(k2); a.v2 = static_cast<const f16*>(v2); a.o = static_cast<bf16*>(o);
    return attention(fill(a), st);
  }
  if (dtype == WD_F32) {
    AttnArgs<float, float> a{};
    a.q = static_cast<const float*>(q); a.k1 = static_cast<const float*>(k1); a.v1 = static_cast<const float*>(v1);
    a.k2 = static_cast<const float*>(k2); a.v2 = static_cast<const float*>(v2); a.o = static_cast<float*>(o);
    return attention(fill(a), st);
  }
  set_error("dtype %d", dtype);
  return WD_ERR_DTYPE;
}

// One key segment with the rows' log-sum-exps, and the merge of two such results.
wd_status wd_attention_lse(int dtype, int batch, int Lq, int heads, int dh, const void* q, const void* k, const void* v,
                           int n, int kv_shared, void* o, float* lse, wd_stream stream) {
  WD_NEED(q); WD_NEED(k); WD_NEED(v); WD_NEED(o); WD_NEED(lse);
  if (batch <= 0 || Lq <= 0 || heads <= 0 || n <= 0) { set_error("attention sizes"); return WD_ERR_SHAPE; }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t D = static_cast<int64_t>(heads) * dh;
  auto fill = [&](auto a) {
    a.q_rs = D; a.kv1_rs = D; a.kv1_bs = kv_shared ? 0 : n * D; a.n1 = n;
    a.o_rs = D; a.batch = batch; a.Lq = Lq; a.heads = heads; a.dh = dh; a.lse = lse;
    return a;
  };
  if (dtype == WD_BF16) {
    AttnArgs<bf16, bf16> a{};
    a.q = static_cast<const bf16*>(q); a.k1 = static_cast<const bf16*>(k); a.v1 = static_cast<const bf16*>(v);
    a.o = static_cast<bf16*>(o);
    return attention(fill(a), st);
  }
  if (dtype == WD_F32) {
    AttnArgs<float, float> a{};
    a.q = static_cast<const float*>(q); a.k1 = static_cast<const float*>(k); a.v1 = static_cast<const float*>(v);
    a.o = static_cast<float*>(o);
    return attention(fill(a), st);
  }
  set_error("wd_attention_lse: dtype %d (WD_BF16 or WD_F32)", dtype);
  return WD_ERR_DTYPE;
}

wd_status wd_attention_fp8_layout(int batch, int64_t Lq, int64_t Lk, int heads, int dh, wd_attn_fp8_layout* out) {
  WD_NEED(out);
  return attn_fp8_layout(batch, Lq, Lk, heads, dh, out);
}

wd_status wd_attention_fp8_quantize(int batch, int64_t Lq, int64_t Lk, int heads, int dh, const void* q, int64_t q_rs,
                                    const void* k, const void* v, int64_t kv_rs, void* buf, size_t buf_bytes,
                                    wd_stream stream) {
  WD_NEED(q); WD_NEED(k); WD_NEED(v); WD_NEED(buf);
  wd_attn_fp8_layout L;
  WD_TRY(attn_fp8_layout(batch, Lq, Lk, heads, dh, &L));
  if (buf_bytes < L.bytes) { set_error("FP8 attention buffer %zu < %zu bytes", buf_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  if (reinterpret_cast<uintptr_t>(buf) & 255u) { set_error("FP8 attention buffer not 256-byte aligned"); return WD_ERR_ALIGN; }
  return attn_fp8_quantize(batch, static_cast<int>(Lq), static_cast<int>(Lk), heads, static_cast<const bf16*>(q), q_rs,
                           static_cast<const bf16*>(k), static_cast<const bf16*>(v), kv_rs, buf, L,
                           static_cast<cudaStream_t>(stream));
}

wd_status wd_attention_fp8(int batch, int64_t Lq, int64_t Lk, int heads, int dh, const void* buf, size_t buf_bytes,
                           void* o, int64_t o_rs, wd_stream stream) {
  WD_NEED(buf); WD_NEED(o);
  wd_attn_fp8_layout L;
  WD_TRY(attn_fp8_layout(batch, Lq, Lk, heads, dh, &L));
  if (buf_bytes < L.bytes) { set_error("FP8 attention buffer %zu < %zu bytes", buf_bytes, L.bytes); return WD_ERR_WORKSPACE; }
  return attn_fp8(batch, static_cast<int>(Lq), static_cast<int>(Lk), heads, buf, L, static_cast<bf16*>(o), o_rs,
                  static_cast<cudaStream_t>(stream));
}

wd_status wd_attention_merge(int dtype, int batch, int Lq, int heads, int dh, float* o_run, float* lse_run,
                             const void* o_part, const float* lse_part, int first, void* out, wd_stream stream) {
  WD_NEED(o_run); WD_NEED(lse_run); WD_NEED(o_part); WD_NEED(lse_part); WD_OPT(out);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == WD_BF16)
    return attn_merge<bf16>(batch, Lq, heads, dh, o_run, lse_run, static_cast<const bf16*>(o_part), lse_part, first,
                            static_cast<bf16*>(out), st);
  if (dtype == WD_F32)
    return attn_merge<float>(batch, Lq, heads, dh, o_run, lse_run, static_cast<const float*>(o_part), lse_part, first,
                             static_cast<float*>(out), st);
  set_error("wd_attention_merge: dtype %d (WD_BF16 or WD_F32)", dtype);
  return WD_ERR_DTYPE;
}

}  // extern "C"
