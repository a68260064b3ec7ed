// k_simt.cu — CUDA-core (FFMA) GEMM and attention.  They serve the fp32
// path, whose 1e-4 parity bar tensor-core tf32 cannot meet, and any bf16
// shape the tensor-core kernels do not cover.  fp32 accumulation throughout.
#include "wd_internal.cuh"

namespace wd {

// ============================================================ epilogue (one element)
template <typename OutT>
__device__ __forceinline__ void epi_one(int mode, const Epi& ep, int64_t m, int n, float acc) {
  const float v = acc + (ep.bias ? ep.bias[n] : 0.f);
  switch (mode) {
    case EPI_STORE: static_cast<OutT*>(ep.out)[m * ep.ldo + n] = from_f<OutT>(v); break;
    case EPI_GELU: static_cast<OutT*>(ep.out)[m * ep.ldo + n] = from_f<OutT>(gelu_erf(v)); break;
    case EPI_F32: static_cast<float*>(ep.out)[m * ep.ldo + n] = v; break;
    case EPI_RESID: {
      float g = 1.f;
      if (ep.gate_a || ep.gate_b) g = (ep.gate_a ? ep.gate_a[n] : 0.f) + (ep.gate_b ? ep.gate_b[n] : 0.f);
      static_cast<float*>(ep.out)[m * ep.ldo + n] += g * v;
      break;
    }
    case EPI_UNPATCH: static_cast<float*>(ep.out)[unpatch_index(ep, m, n)] = v; break;
    case EPI_STORE_F16: static_cast<f16*>(ep.out)[m * ep.ldo + n] = __float2half_rn(v); break;
  }
}

// ============================================================ GEMM
// 64x64 output tile per 256-thread CTA, 4x4 per thread, K staged 16 at a time.
template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(int M, int N, int K, const T* __restrict__ A, int64_t lda,
                                                   const T* __restrict__ B, int64_t ldb, int mode, Epi ep) {
  constexpr int BM = 64, BN = 64, BK = 16, PAD = 4;
  __shared__ __align__(16) float As[BK][BM + PAD];
  __shared__ __align__(16) float Bs[BK][BN + PAD];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int idx = tid + r * 256, row = idx >> 4, kk = idx & 15;
      const int64_t gm = m0 + row;
      const int gn = n0 + row, gk = k0 + kk;
      As[kk][row] = (gm < M && gk < K) ? to_f<T>(A[gm * lda + gk]) : 0.f;
      Bs[kk][row] = (gn < N && gk < K) ? to_f<T>(B[static_cast<int64_t>(gn) * ldb + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) epi_one<T>(mode, ep, m, n, acc[i][j]);
    }
  }
}

template <typename T>
wd_status gemm_simt(int M, int N, int K, const T* A, int64_t lda, const T* B, int64_t ldb, int mode, const Epi& ep,
                    cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) { set_error("gemm: empty shape %d x %d x %d", M, N, K); return WD_ERR_SHAPE; }
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  if (grid.y > 65535u) { set_error("gemm_simt: M=%d too large", M); return WD_ERR_SHAPE; }
  Trace tr(KC_GEMM, st);
  k_gemm_simt<T><<<grid, 256, 0, st>>>(M, N, K, A, lda, B, ldb, mode, ep);
  return launch_status("gemm_simt");
}
template wd_status gemm_simt<float>(int, int, int, const float*, int64_t, const float*, int64_t, int, const Epi&,
                                   cudaStream_t);
template wd_status gemm_simt<bf16>(int, int, int, const bf16*, int64_t, const bf16*, int64_t, int, const Epi&,
                                  cudaStream_t);

// ============================================================ attention
// Flash-style: a CTA owns 64 query rows of one (batch, head) and streams
// 64-key tiles through shared memory with an online softmax (exp2, log2(e)/
// sqrt(dh) folded into q).  A second key/value segment, when present, gets its
// own softmax and is added after normalisation ("图解 Wan2.1 I2V" 5.4).
template <typename T, typename TO, int DH>
__global__ void __launch_bounds__(256) k_attn_simt(AttnArgs<T, TO> a, float qscale) {
  constexpr int BQ = 64, BK = 64, P = 68, CW = DH / 16;
  extern __shared__ __align__(16) float sm[];
  float* Qt = sm;               // [DH][P]  q transposed
  float* Kt = Qt + DH * P;      // [DH][P]  k transposed
  float* Vs = Kt + DH * P;      // [BK][DH]
  float* Pt = Vs + BK * DH;     // [BK][P]  probabilities transposed
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int q0 = blockIdx.x * BQ, h = blockIdx.y, b = blockIdx.z;
  for (int idx = tid; idx < BQ * DH; idx += 256) {
    const int i = idx / DH, d = idx % DH, l = q0 + i;
    Qt[d * P + i] = l < a.Lq ? to_f<T>(a.q[(static_cast<int64_t>(b) * a.Lq + l) * a.q_rs + h * DH + d]) * qscale : 0.f;
  }
  float out[4][CW] = {};
  for (int seg = 0; seg < 2; ++seg) {
    const T* K = seg ? a.k2 : a.k1;
    const T* V = seg ? a.v2 : a.v1;
    if (K == nullptr) break;
    const int n = seg ? a.n2 : a.n1;
    const int64_t rs = seg ? a.kv2_rs : a.kv1_rs;
    const int64_t base = (seg ? a.kv2_bs : a.kv1_bs) * b + static_cast<int64_t>(h) * DH;
    float o[4][CW] = {};
    float mrow[4], lrow[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { mrow[i] = -INFINITY; lrow[i] = 0.f; }
    for (int k0 = 0; k0 < n; k0 += BK) {
      __syncthreads();
      for (int idx = tid; idx < BK * DH; idx += 256) {
        const int j = idx / DH, d = idx % DH, key = k0 + j;
        float kv = 0.f, vv = 0.f;
        if (key < n) {
          kv = to_f<T>(K[base + key * rs + d]);
          vv = to_f<T>(V[base + key * rs + d]);
        }
        Kt[d * P + j] = kv;
        Vs[j * DH + d] = vv;
      }
      __syncthreads();
      float s[4][4] = {};
#pragma unroll 8
      for (int d = 0; d < DH; ++d) {
        const float4 qv = *reinterpret_cast<const float4*>(&Qt[d * P + ty * 4]);
        const float4 kv = *reinterpret_cast<const float4*>(&Kt[d * P + tx * 4]);
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) s[i][j] = fmaf(qa[i], ka[j], s[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (k0 + tx * 4 + j >= n) s[i][j] = -INFINITY;
          mx = fmaxf(mx, s[i][j]);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mnew = fmaxf(mrow[i], mx);
        const float alpha = exp2f(mrow[i] - mnew);
        float rs_ = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s[i][j] = exp2f(s[i][j] - mnew);
          rs_ += s[i][j];
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) rs_ += __shfl_xor_sync(0xffffffffu, rs_, off);
        lrow[i] = lrow[i] * alpha + rs_;
        mrow[i] = mnew;
#pragma unroll
        for (int c = 0; c < CW; ++c) o[i][c] *= alpha;
#pragma unroll
        for (int j = 0; j < 4; ++j) Pt[(tx * 4 + j) * P + ty * 4 + i] = s[i][j];
      }
      __syncthreads();
#pragma unroll 4
      for (int j = 0; j < BK; ++j) {
        const float4 pv = *reinterpret_cast<const float4*>(&Pt[j * P + ty * 4]);
        const float pa[4] = {pv.x, pv.y, pv.z, pv.w};
        float vv[CW];
#pragma unroll
        for (int c = 0; c < CW; ++c) vv[c] = Vs[j * DH + tx * CW + c];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int c = 0; c < CW; ++c) o[i][c] = fmaf(pa[i], vv[c], o[i][c]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float inv = 1.f / lrow[i];
#pragma unroll
      for (int c = 0; c < CW; ++c) out[i][c] += o[i][c] * inv;
      // one segment: the row's log-sum-exp in log2 units (the scores carry log2(e) already)
      const int l = q0 + ty * 4 + i;
      if (a.lse && !a.k2 && tx == 0 && l < a.Lq)
        a.lse[(static_cast<int64_t>(b) * a.heads + h) * a.Lq + l] = mrow[i] + log2f(lrow[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int l = q0 + ty * 4 + i;
    if (l >= a.Lq) continue;
    TO* dst = a.o + (static_cast<int64_t>(b) * a.Lq + l) * a.o_rs + h * DH + tx * CW;
#pragma unroll
    for (int c = 0; c < CW; ++c) dst[c] = from_f<TO>(out[i][c]);
  }
}

template <typename T, typename TO, int DH>
static wd_status launch_attn_simt(const AttnArgs<T, TO>& a, cudaStream_t st) {
  const size_t smem = (2 * DH * 68 + 64 * DH + 64 * 68) * sizeof(float);
  static bool attr_set[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set[dev & 15]) {
    cudaFuncSetAttribute(k_attn_simt<T, TO, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    attr_set[dev & 15] = true;
  }
  dim3 grid((a.Lq + 63) / 64, a.heads, a.batch);
  const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(DH));
  Trace tr(a.cross ? KC_ATTN_CROSS : KC_ATTN_SELF, st);
  k_attn_simt<T, TO, DH><<<grid, 256, smem, st>>>(a, qscale);
  return launch_status("attention_simt");
}

template <typename T, typename TO>
wd_status attention_simt(const AttnArgs<T, TO>& a, cudaStream_t st) {
  if (a.n1 <= 0 || (a.k2 && a.n2 <= 0)) { set_error("attention: empty key segment"); return WD_ERR_SHAPE; }
  switch (a.dh) {
    case 32: return launch_attn_simt<T, TO, 32>(a, st);
    case 64: return launch_attn_simt<T, TO, 64>(a, st);
    case 128: return launch_attn_simt<T, TO, 128>(a, st);
    default: set_error("attention: head dim %d not supported (32, 64, 128)", a.dh); return WD_ERR_SHAPE;
  }
}
template wd_status attention_simt<float, float>(const AttnArgs<float, float>&, cudaStream_t);
template wd_status attention_simt<bf16, bf16>(const AttnArgs<bf16, bf16>&, cudaStream_t);
template wd_status attention_simt<f16, bf16>(const AttnArgs<f16, bf16>&, cudaStream_t);

}  // namespace wd
