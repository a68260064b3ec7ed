// wd_internal.cuh — declarations shared by the kernels of libwd (one
// translation unit: wd_lib.cu includes every kernel file).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>
#include <cstdio>
#include <string>

#include "../../include/wd.h"
#include "wd_ptx.cuh"

namespace wd {

using bf16 = __nv_bfloat16;
using f16 = __half;

// ------------------------------------------------------------------ errors
void set_error(const char* fmt, ...);

#define WD_TRY(expr)                       \
  do {                                     \
    wd_status _s = (expr);                 \
    if (_s != WD_OK) return _s;            \
  } while (0)

wd_status launch_status(const char* what);   // cudaGetLastError -> WD_ERR_CUDA + message

// ------------------------------------------------------------------ tracing
// Kernel classes for launch accounting (same order as wd_kernel_class in wd.h).
enum KClass : int { KC_GEMM = 0, KC_ATTN_SELF = 1, KC_ATTN_CROSS = 2, KC_NORM = 3, KC_ROPE = 4, KC_EULER = 5,
                    KC_SMALL = 6, KC_COUNT = 7 };
// Scope guard around one launch: counts it and, with timing on, records an
// event on `st` at construction and another at destruction.
struct Trace {
  Trace(int cls, cudaStream_t st);
  ~Trace();
  int cls_;
  cudaStream_t st_;
  int slot_;
};

// ------------------------------------------------------------------ element conversions
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f<f16>(f16 v) { return __half2float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ f16 from_f<f16>(float v) { return __float2half_rn(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// Exact GELU x * Phi(x) (erf form).
__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

// GELU for the tensor-core GEMM epilogue: x * Phi(x) with the tail probability
// E = erfc(|x| / sqrt 2) / 2 from the rational approximation of Abramowitz and
// Stegun, Handbook of Mathematical Functions, 7.1.26 (Hastings):
//   erfc(y) = t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-y^2),  t = 1 / (1 + p y),
// |error| <= 1.5e-7 for y >= 0; the a_i below are the published ones halved.
// Phi(x) = 1 - E for x >= 0 and E for x < 0, so the negative tail is never a
// difference of nearly equal numbers.  Two MUFU operations (reciprocal, 2^x)
// and twelve FMA-pipe ones per value (about seven in the packed form below),
// against about thirty issue slots for the erff form.
__device__ __forceinline__ float gelu_as(float x) {
  float t, e;
  const float y = fabsf(x) * 0.70710678118654752f;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, y, 1.0f)));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * y * y));
  const float poly =
      t * fmaf(fmaf(fmaf(fmaf(0.5307027145f, t, -0.7265760135f), t, 0.7107068705f), t, -0.142248368f), t, 0.127414796f);
  const float tail = poly * e;
  return x * (x >= 0.f ? 1.0f - tail : tail);
}
// gelu_as on two values with the packed fp32 instructions (f32x2): the same
// operations and roundings on each lane, in fewer instructions.
__device__ __forceinline__ float2 gelu_as2(float2 x) {
  auto bc = [](float c) { return make_float2(c, c); };
  const float2 y = fmul2(make_float2(fabsf(x.x), fabsf(x.y)), bc(0.70710678118654752f));
  const float2 den = ffma2(bc(0.3275911f), y, bc(1.0f));
  const float2 z = fmul2(fmul2(bc(-1.4426950408889634f), y), y);
  float2 t, e;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t.x) : "f"(den.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t.y) : "f"(den.y));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.x) : "f"(z.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.y) : "f"(z.y));
  const float2 poly = fmul2(
      t, ffma2(ffma2(ffma2(ffma2(bc(0.5307027145f), t, bc(-0.7265760135f)), t, bc(0.7107068705f)), t, bc(-0.142248368f)),
               t, bc(0.127414796f)));
  const float2 tail = fmul2(poly, e);
  const float2 one_m = fsub2(bc(1.0f), tail);
  return fmul2(x, make_float2(x.x >= 0.f ? one_m.x : tail.x, x.y >= 0.f ? one_m.y : tail.y));
}

// ------------------------------------------------------------------ GEMM epilogues
// Every GEMM computes acc[m, n] = sum_k A[m, k] * B[n, k] (B is a Linear weight
// [out, in]) and then one of these epilogues, with v = acc + bias[n]:
enum EpiMode : int {
  EPI_STORE = 0,      // out[m, n] = v                        (out in the activation type)
  EPI_GELU = 1,       // out[m, n] = GELU(v)                  (out in the activation type)
  EPI_F32 = 2,        // out[m, n] = v                        (out fp32)
  EPI_RESID = 3,      // out[m, n] += g[n] * v, g = ga + gb   (out fp32 residual, in place)
  EPI_UNPATCH = 4,    // unpatchify scatter of v into [B, 16, T, H, W] fp32
  EPI_STORE_F16 = 5,  // out[m, n] = v                        (out IEEE half: cross-attention operands)
};

struct Epi {
  void* out;
  int64_t ldo;            // row stride of out, elements (unused by EPI_UNPATCH)
  const float* bias;      // [N] or null
  const float* gate_a;    // EPI_RESID: gate = gate_a[n] + gate_b[n]; both null -> 1
  const float* gate_b;
  int T, Hp, Wp, L;       // EPI_UNPATCH geometry
  const float* sa;        // FP8 GEMM: acc[m, n] is scaled by sa[m] * sb[n] before the bias; null otherwise
  const float* sb;
};

// Unpatchify address of GEMM element (row m = b*L + l, column n = c*4+kh*2+kw).
__device__ __forceinline__ int64_t unpatch_index(const Epi& ep, int64_t m, int n) {
  const int64_t b = m / ep.L;
  const int l = static_cast<int>(m - b * ep.L);
  const int x = l % ep.Wp, y = (l / ep.Wp) % ep.Hp, f = l / (ep.Wp * ep.Hp);
  const int c = n >> 2, kh = (n >> 1) & 1, kw = n & 1;
  const int H = 2 * ep.Hp, W = 2 * ep.Wp;
  return (((b * 16 + c) * ep.T + f) * H + (2 * y + kh)) * static_cast<int64_t>(W) + (2 * x + kw);
}

// ------------------------------------------------------------------ internal launchers
// C = epilogue(A[M,K] * B[N,K]^T): A, B in T (float or bf16).
template <typename T>
wd_status gemm_simt(int M, int N, int K, const T* A, int64_t lda, const T* B, int64_t ldb, int mode,
                    const Epi& ep, cudaStream_t st);
// Tensor-core (tcgen05 + TMA) bf16 GEMM.
wd_status gemm_tc(int M, int N, int K, const bf16* A, int64_t lda, const bf16* B, int64_t ldb, int mode,
                  const Epi& ep, cudaStream_t st);
// The same with e4m3 operands (one byte each; lda, ldb in elements = bytes) and the
// scales ep.sa[M], ep.sb[N] applied to the fp32 accumulator.
wd_status gemm_tc_fp8(int M, int N, int K, const uint8_t* A, int64_t lda, const uint8_t* B, int64_t ldb, int mode,
                      const Epi& ep, cudaStream_t st);
// Per-row e4m3 quantisation: scale[r] = amax_r / 448, q[r, k] = e4m3(x[r, k] / scale[r]).
template <typename T>
wd_status quant_rows_e4m3(int rows, int K, const T* x, uint8_t* q, float* scale, cudaStream_t st);

// Multi-head attention O = softmax(Q K^T / sqrt(dh)) V per (batch, head),
// optionally summed with a second, independently normalised key/value
// segment (the decoupled image/text cross-attention).  TI is the type of
// q, k and v; TO the type of o (the bf16 path's cross-attention reads IEEE
// half operands and writes bf16).
template <typename TI, typename TO = TI>
struct AttnArgs {
  const TI* q; int64_t q_rs;                   // q row (b, l): q + (b*Lq + l)*q_rs + h*dh
  const TI* k1; const TI* v1; int64_t kv1_rs; int64_t kv1_bs; int n1;
  const TI* k2; const TI* v2; int64_t kv2_rs; int64_t kv2_bs; int n2;   // k2 == null: one segment
  TO* o; int64_t o_rs;
  int batch, Lq, heads, dh;
  bool cross;                                  // counted as cross-attention in the launch trace
  // one segment only, optional: lse[(b*heads + h)*Lq + l] = log2 sum_j 2^(q k_j^T log2(e) / sqrt(dh)),
  // the row's log-sum-exp in log2 units (for merging attentions over parts of the keys)
  float* lse;
};
// Merge of attentions over disjoint key sets (the ring level of sequence parallelism):
// o_run, lse_run (fp32, [batch, Lq, heads*dh] and [batch, heads, Lq]) absorb the part
// (o_part in TP, lse_part); first: the part is copied; out (TP, optional): the merged
// output rounded to TP.
template <typename TP>
wd_status attn_merge(int batch, int Lq, int heads, int dh, float* o_run, float* lse_run, const TP* o_part,
                     const float* lse_part, int first, TP* out, cudaStream_t st);
template <typename TI, typename TO>
wd_status attention_simt(const AttnArgs<TI, TO>& a, cudaStream_t st);
// Tensor-core attention (dh = 128; other head sizes go to attention_simt).
wd_status attention_tc(const AttnArgs<bf16, bf16>& a, cudaStream_t st);
wd_status attention_tc(const AttnArgs<f16, bf16>& a, cudaStream_t st);
// FP8 attention (k_attn_f8.cu): the operand buffer's layout, the quantisation
// of bf16 q, k, v into it and the attention on it (bf16 output).
wd_status attn_fp8_layout(int batch, int64_t Lq, int64_t Lk, int heads, int dh, wd_attn_fp8_layout* L);
wd_status attn_fp8_quantize(int batch, int Lq, int Lk, int heads, const bf16* q, int64_t q_rs, const bf16* k,
                            const bf16* v, int64_t kv_rs, void* buf, const wd_attn_fp8_layout& L, cudaStream_t st);
wd_status attn_fp8(int batch, int Lq, int Lk, int heads, const void* buf, const wd_attn_fp8_layout& L, bf16* o,
                   int64_t o_rs, cudaStream_t st);

}  // namespace wd
