// k_small.cu — the bandwidth-bound and latency-bound kernels of the step:
// conditioning y, CFG Euler update, shared time MLP, adaLN norm+modulate,
// QK-RMSNorm + 3D RoPE, the patch gather feeding the patch-embed GEMM, and
// the per-row e4m3 quantisation feeding the FP8 GEMM.
#include "wd_internal.cuh"

#include <cuda_fp8.h>

namespace wd {

// ============================================================ conditioning y
// y[0:4] = temporal mask, y[4:20] = image latent ("图解 Wan2.1 I2V" 4.1).
// The mask value of (channel c, latent frame f) is bit (f*4 + c) of `bits`.
struct MaskBits {
  uint32_t w[32];   // up to 1024 (channel, frame) entries: T <= 256
};

__global__ void k_cond_y(const float* __restrict__ img, MaskBits mb, int T, int64_t HW, float* __restrict__ y) {
  const int64_t plane = static_cast<int64_t>(T) * HW;    // one channel
  const int64_t n = 20 * plane;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i / plane);
    if (c < 4) {
      const int f = static_cast<int>((i - c * plane) / HW);
      const int bit = f * 4 + c;
      y[i] = ((mb.w[bit >> 5] >> (bit & 31)) & 1u) ? 1.0f : 0.0f;
    } else {
      y[i] = img[i - 4 * plane];
    }
  }
}

// ============================================================ CFG Euler step
// x += dt * (vu + s * (vc - vu))   ("图解 Wan2.1 I2V" 7; Wan 技术深度解析 2.7).
// 16 B per element of traffic; float4 vectors, grid-stride over the tensor.
__global__ void __launch_bounds__(256) k_euler_cfg(float* __restrict__ x, const float* __restrict__ vc,
                                                   const float* __restrict__ vu, float s, float dt, int64_t n) {
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* c4 = reinterpret_cast<const float4*>(vc);
  const float4* u4 = reinterpret_cast<const float4*>(vu);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    float4 a = x4[i];
    const float4 c = __ldcs(c4 + i);
    if (vu != nullptr) {
      const float4 u = __ldcs(u4 + i);
      a.x += dt * (u.x + s * (c.x - u.x));
      a.y += dt * (u.y + s * (c.y - u.y));
      a.z += dt * (u.z + s * (c.z - u.z));
      a.w += dt * (u.w + s * (c.w - u.w));
    } else {
      a.x += dt * c.x; a.y += dt * c.y; a.z += dt * c.z; a.w += dt * c.w;
    }
    x4[i] = a;
  }
  // scalar tail
  for (int64_t i = 4 * n4 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride) {
    const float v = vu != nullptr ? vu[i] + s * (vc[i] - vu[i]) : vc[i];
    x[i] += dt * v;
  }
}

// ============================================================ time MLP
// One warp per output row: out[o] = sum_i W[o, i] * in(i) + b[o], where in(i)
// is the 256-wide sinusoid of tau (mode 0) or SiLU(x[i]) (mode 1).
// Sinusoid ("图解 Wan2.1 I2V" 5.2): [cos(tau w_i), sin(tau w_i)],
// w_i = 10000^(-i/128); the angle is formed in double because tau reaches 1000.
__device__ __forceinline__ float time_input(int mode, const float* x, float tau, int i) {
  if (mode == 0) {
    const int j = i & 127;
    const double a = static_cast<double>(tau) * pow(10000.0, -static_cast<double>(j) / 128.0);
    return static_cast<float>(i < 128 ? cos(a) : sin(a));
  }
  const float v = x[i];
  return v / (1.0f + expf(-v));
}

__global__ void __launch_bounds__(256) k_time_matvec(const float* __restrict__ W, const float* __restrict__ b,
                                                     const float* __restrict__ x, float tau, int mode, int O, int I,
                                                     float* __restrict__ out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= O) return;
  const float* w = W + static_cast<int64_t>(warp) * I;
  float acc = 0.f;
  for (int i = lane; i < I; i += 32) acc += w[i] * time_input(mode, x, tau, i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) out[warp] = acc + b[warp];
}

// ============================================================ norm + modulate
// out = norm(x) * mul + add, per row of the fp32 residual stream, where either
//   mul = 1 + (sc_a + sc_b), add = sh_a + sh_b      (adaLN, "图解 Wan2.1 I2V" 5.2)
//   mul = gamma, add = beta                         (affine LayerNorm)
// norm = LayerNorm (no affine) or RMSNorm.  One warp per row; each lane holds
// NV float4 of the row in registers (D = 128 * NV), so x is read once.
// OutT = uint8_t: the row is quantised to e4m3 as by k_quant_rows_e4m3 (scale =
// amax / 448, codes e4m3(v / scale), IEEE division, saturating), from the fp32
// values, and the scale written to scale[row] (the FP8 block's GEMM inputs).
struct NormArgs {
  const float* x;
  int64_t rows;
  int D;
  const float *sh_a, *sh_b, *sc_a, *sc_b;   // adaLN vectors (any may be null = 0)
  const float *gamma, *beta;                // affine (used when gamma != null)
  int rms;
  float eps;
  void* out;
  float* scale;                             // OutT = uint8_t: per-row e4m3 scales
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4_or0(const float* p, int i) {
  return p ? *reinterpret_cast<const float4*>(p + i) : make_float4(0.f, 0.f, 0.f, 0.f);
}

template <typename OutT, int NV>
__global__ void __launch_bounds__(256) k_norm_mod(NormArgs a) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  const float* x = a.x + row * a.D;
  float4 v[NV];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    v[i] = __ldcs(reinterpret_cast<const float4*>(x) + i * 32 + lane);
    s += v[i].x + v[i].y + v[i].z + v[i].w;
  }
  float mean = 0.f;
  if (!a.rms) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    mean = s / a.D;
  }
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const float dx = v[i].x - mean, dy = v[i].y - mean, dz = v[i].z - mean, dw = v[i].w - mean;
    q += dx * dx + dy * dy + dz * dz + dw * dw;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / a.D + a.eps);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane) * 4;
    float4 mul, add;
    if (a.gamma) {
      mul = ld4(a.gamma + c);
      add = ld4_or0(a.beta, c);
    } else {
      const float4 p = ld4_or0(a.sc_a, c), r = ld4_or0(a.sc_b, c);
      const float4 h = ld4_or0(a.sh_a, c), g = ld4_or0(a.sh_b, c);
      mul = make_float4(1.f + p.x + r.x, 1.f + p.y + r.y, 1.f + p.z + r.z, 1.f + p.w + r.w);
      add = make_float4(h.x + g.x, h.y + g.y, h.z + g.z, h.w + g.w);
    }
    const float o0 = (v[i].x - mean) * rstd * mul.x + add.x;
    const float o1 = (v[i].y - mean) * rstd * mul.y + add.y;
    const float o2 = (v[i].z - mean) * rstd * mul.z + add.z;
    const float o3 = (v[i].w - mean) * rstd * mul.w + add.w;
    if constexpr (std::is_same<OutT, uint8_t>::value) {   // kept for the quantisation below
      v[i] = make_float4(o0, o1, o2, o3);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(o0), fabsf(o1)), fmaxf(fabsf(o2), fabsf(o3))));
    } else if constexpr (sizeof(OutT) == 2) {
      uint2 pk = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
      *reinterpret_cast<uint2*>(static_cast<bf16*>(a.out) + row * a.D + c) = pk;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * a.D + c) = make_float4(o0, o1, o2, o3);
    }
  }
  if constexpr (std::is_same<OutT, uint8_t>::value) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = (i * 32 + lane) * 4;
      const float e[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t w = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(e[j], sc), __NV_SATFINITE, __NV_E4M3)) << (8 * j);
      *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.out) + row * a.D + c) = w;
    }
    if (lane == 0) a.scale[row] = sc;
  }
}

template <typename OutT>
wd_status norm_mod(const NormArgs& a, cudaStream_t st) {
  if (a.D % 128 != 0) { set_error("norm: D=%d must be a multiple of 128", a.D); return WD_ERR_SHAPE; }
  const unsigned grid = static_cast<unsigned>((a.rows * 32 + 255) / 256);
  Trace tr(KC_NORM, st);
  switch (a.D / 128) {
    case 1: k_norm_mod<OutT, 1><<<grid, 256, 0, st>>>(a); break;
    case 2: k_norm_mod<OutT, 2><<<grid, 256, 0, st>>>(a); break;
    case 4: k_norm_mod<OutT, 4><<<grid, 256, 0, st>>>(a); break;
    case 8: k_norm_mod<OutT, 8><<<grid, 256, 0, st>>>(a); break;
    case 12: k_norm_mod<OutT, 12><<<grid, 256, 0, st>>>(a); break;
    case 16: k_norm_mod<OutT, 16><<<grid, 256, 0, st>>>(a); break;
    case 24: k_norm_mod<OutT, 24><<<grid, 256, 0, st>>>(a); break;
    case 32: k_norm_mod<OutT, 32><<<grid, 256, 0, st>>>(a); break;
    case 40: k_norm_mod<OutT, 40><<<grid, 256, 0, st>>>(a); break;
    default: set_error("norm: D=%d not instantiated", a.D); return WD_ERR_SHAPE;
  }
  return launch_status("norm_mod");
}

// ============================================================ 3D RoPE table
// tab[axis][p][j] = (cos, sin) of p * 10000^(-2 j_s / d_s) for every pair j of
// a head whose segment (frame / row / column, sizes dh-4(dh/6), 2(dh/6),
// 2(dh/6), "图解 Wan2.1 I2V" 5.3) is `axis`; j_s counts pairs inside the segment.
// Rows: axis 0 has T positions, axis 1 Hp, axis 2 Wp, stacked.
__global__ void k_rope_table(float2* tab, int T, int Hp, int Wp, int dh) {
  const int half = dh / 2;
  const int s6 = dh / 6, dT = dh - 4 * s6, dH = 2 * s6;
  const int rows = T + Hp + Wp;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * half; i += gridDim.x * blockDim.x) {
    const int r = i / half, j = i % half;
    const int axis = r < T ? 0 : (r < T + Hp ? 1 : 2);
    const int p = r - (axis == 0 ? 0 : (axis == 1 ? T : T + Hp));
    const int d = 2 * j;
    const int seg = d < dT ? 0 : (d < dT + dH ? 1 : 2);
    float2 cs = make_float2(1.f, 0.f);
    if (seg == axis) {
      const int off = seg == 0 ? 0 : (seg == 1 ? dT : dT + dH);
      const int size = seg == 0 ? dT : dH;
      const double th = static_cast<double>(p) * pow(10000.0, -static_cast<double>(d - off) / size);
      cs = make_float2(static_cast<float>(cos(th)), static_cast<float>(sin(th)));
    }
    tab[i] = cs;
  }
}

// ============================================================ QK-RMSNorm + 3D RoPE
// In place on the fused projection buffer qkv [rows, 3D]: q = cols [0, D),
// k = cols [D, 2D).  q <- RoPE(RMSNorm_D(q) * g_q), k likewise
// ("图解 Wan2.1 I2V" 5.3 (1) and (2)).  The rows are batch x n_tok tokens of a
// slice that starts at token tok0 of the sequence (the whole sequence: tok0
// = 0, n_tok = L), so row r holds token tok0 + r % n_tok.  One warp per
// (row, q|k); each lane owns NC chunks of 4 channels (2 rotation pairs), so
// the row sits in registers between the norm and the rotation.
template <typename T, int NC>
__global__ void __launch_bounds__(256) k_qknorm_rope(T* qkv, int64_t rows, int D, int dh, int n_tok, int tok0, int Hp,
                                                     int Wp, int T_, const float* __restrict__ gq,
                                                     const float* __restrict__ gk, const float2* __restrict__ tab,
                                                     float eps) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= 2 * rows) return;
  const int64_t row = w >> 1;
  const int which = static_cast<int>(w & 1);
  T* p = qkv + row * 3 * static_cast<int64_t>(D) + which * D;
  const float* g = which ? gk : gq;
  float v[NC][4];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = (i * 32 + lane) * 4;
    if constexpr (sizeof(T) == 2) {
      const uint2 u = *reinterpret_cast<const uint2*>(p + c);
      const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
      v[i][0] = a.x; v[i][1] = a.y; v[i][2] = b.x; v[i][3] = b.y;
    } else {
      const float4 a = *reinterpret_cast<const float4*>(p + c);
      v[i][0] = a.x; v[i][1] = a.y; v[i][2] = a.z; v[i][3] = a.w;
    }
    ss += v[i][0] * v[i][0] + v[i][1] * v[i][1] + v[i][2] * v[i][2] + v[i][3] * v[i][3];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / D + eps);
  const int l = tok0 + static_cast<int>(row % n_tok);   // the token's index in the whole sequence
  const int px = l % Wp, py = (l / Wp) % Hp, pf = l / (Wp * Hp);
  const int half = dh / 2;
  const int s6 = dh / 6, dT = dh - 4 * s6, dH = 2 * s6;
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    const int c = (i * 32 + lane) * 4;
    const float4 gg = *reinterpret_cast<const float4*>(g + c);
    const float n0 = v[i][0] * r * gg.x, n1 = v[i][1] * r * gg.y, n2 = v[i][2] * r * gg.z, n3 = v[i][3] * r * gg.w;
    float out[4];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int d = (c % dh) + 2 * pr;
      const int j = d >> 1;
      const int trow = d < dT ? pf : (d < dT + dH ? T_ + py : T_ + Hp + px);
      const float2 cs = tab[trow * half + j];
      const float re = pr ? n2 : n0, im = pr ? n3 : n1;
      out[2 * pr] = re * cs.x - im * cs.y;
      out[2 * pr + 1] = re * cs.y + im * cs.x;
    }
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint2*>(p + c) = make_uint2(pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]));
    } else {
      *reinterpret_cast<float4*>(p + c) = make_float4(out[0], out[1], out[2], out[3]);
    }
  }
}

template <typename T>
wd_status qknorm_rope(T* qkv, int64_t rows, const wd_dims& d, const float* gq, const float* gk, const float2* tab,
                      int64_t n_tok, int64_t tok0, cudaStream_t st) {
  const int D = d.D, dh = D / d.heads;
  const unsigned grid = static_cast<unsigned>((2 * rows * 32 + 255) / 256);
  const int nt = static_cast<int>(n_tok), t0 = static_cast<int>(tok0);
  Trace tr(KC_ROPE, st);
#define WD_QKR(NC)                                                                                            \
  k_qknorm_rope<T, NC><<<grid, 256, 0, st>>>(qkv, rows, D, dh, nt, t0, d.H / 2, d.W / 2, d.T, gq, gk, tab, d.eps); \
  break;
  switch (D / 128) {
    case 1: WD_QKR(1)
    case 2: WD_QKR(2)
    case 4: WD_QKR(4)
    case 8: WD_QKR(8)
    case 12: WD_QKR(12)
    case 16: WD_QKR(16)
    case 24: WD_QKR(24)
    case 32: WD_QKR(32)
    case 40: WD_QKR(40)
    default: set_error("qknorm_rope: D=%d not instantiated", D); return WD_ERR_SHAPE;
  }
#undef WD_QKR
  return launch_status("qknorm_rope");
}

// ============================================================ patch gather
// a[m, k] for m = b*L + l and k = c*4 + kh*2 + kw: the (1,2,2) receptive field
// of token l in the 36-channel input concat(x_t[16], y[20]) (K = 144,
// "图解 Wan2.1 I2V" 4.2 and 5.1; y is shared by the batch), or in x_t alone
// for the text-to-video model (K = 64, section 9 of the same page).
template <typename T>
__global__ void __launch_bounds__(256) k_patch_gather(const float* __restrict__ xt, const float* __restrict__ y, int B,
                                                      int Tn, int H, int W, int K, T* __restrict__ a) {
  const int Hp = H / 2, Wp = W / 2;
  const int64_t L = static_cast<int64_t>(Tn) * Hp * Wp;
  const int64_t n = static_cast<int64_t>(B) * L * K;
  const int64_t HW = static_cast<int64_t>(H) * W, plane = Tn * HW;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int k = static_cast<int>(i % K);
    const int64_t m = i / K;
    const int64_t b = m / L;
    const int l = static_cast<int>(m - b * L);
    const int x = l % Wp, yy = (l / Wp) % Hp, f = l / (Wp * Hp);
    const int c = k >> 2, kh = (k >> 1) & 1, kw = k & 1;
    const int64_t off = f * HW + (2 * yy + kh) * static_cast<int64_t>(W) + (2 * x + kw);
    const float v = c < 16 ? xt[(b * 16 + c) * plane + off] : y[(c - 16) * plane + off];
    a[i] = from_f<T>(v);
  }
}


// ============================================================ merging attention over key parts
// For a query row, the attention over the union of disjoint key sets is the
// average of the attentions over each set weighted by each set's share of the
// softmax denominator: with row log-sum-exps lse_r, lse_p (log2 units) and
// M = max(lse_r, lse_p), o = (2^(lse_r - M) o_r + 2^(lse_p - M) o_p) / (2^(lse_r - M) + 2^(lse_p - M))
// and lse = M + log2(2^(lse_r - M) + 2^(lse_p - M)).  One warp per (batch, head, row).
template <typename TP>
__global__ void __launch_bounds__(256) k_attn_merge(int batch, int Lq, int heads, int dh, float* __restrict__ o_run,
                                                    float* __restrict__ lse_run, const TP* __restrict__ o_part,
                                                    const float* __restrict__ lse_part, int first, TP* __restrict__ out) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;   // (b, h, l)
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(batch) * heads * Lq) return;
  const int l = static_cast<int>(w % Lq);
  const int64_t bh = w / Lq;
  const int h = static_cast<int>(bh % heads);
  const int64_t b = bh / heads;
  const int64_t base = (b * Lq + l) * static_cast<int64_t>(heads) * dh + static_cast<int64_t>(h) * dh;
  const float lp = lse_part[w];
  float wr = 0.f, wp = 1.f, lnew = lp;
  if (!first) {
    const float lr = lse_run[w];
    const float M = fmaxf(lr, lp);
    const float a = exp2f(lr - M), c = exp2f(lp - M), sum = a + c;
    wr = a / sum;
    wp = c / sum;
    lnew = M + log2f(sum);
  }
  for (int d = lane; d < dh; d += 32) {
    const float v = (first ? 0.f : wr * o_run[base + d]) + wp * to_f<TP>(o_part[base + d]);
    o_run[base + d] = v;
    if (out) out[base + d] = from_f<TP>(v);
  }
  __syncwarp();
  if (lane == 0) lse_run[w] = lnew;
}

template <typename TP>
wd_status attn_merge(int batch, int Lq, int heads, int dh, float* o_run, float* lse_run, const TP* o_part,
                     const float* lse_part, int first, TP* out, cudaStream_t st) {
  if (batch <= 0 || Lq <= 0 || heads <= 0 || dh <= 0) { set_error("attention merge: empty shape"); return WD_ERR_SHAPE; }
  const int64_t threads = static_cast<int64_t>(batch) * heads * Lq * 32;
  Trace tr(KC_SMALL, st);
  k_attn_merge<TP><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(batch, Lq, heads, dh, o_run, lse_run,
                                                                               o_part, lse_part, first, out);
  return launch_status("attention_merge");
}
template wd_status attn_merge<bf16>(int, int, int, int, float*, float*, const bf16*, const float*, int, bf16*,
                                    cudaStream_t);
template wd_status attn_merge<float>(int, int, int, int, float*, float*, const float*, const float*, int, float*,
                                     cudaStream_t);

// ============================================================ e4m3 row quantisation
// One warp per row: amax over the row, scale = amax / 448 (IEEE division), then
// q = e4m3(x / scale) with round-to-nearest-even and saturation at +-448 (the
// FP8 GEMM of "Wan（通义万相）..." 5.3 with per-token / per-channel scales).
// Each lane converts 8 consecutive elements per pass; K is a multiple of 8.
template <typename T>
__global__ void __launch_bounds__(256) k_quant_rows_e4m3(const T* __restrict__ x, int rows, int K,
                                                          uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* xr = x + static_cast<int64_t>(row) * K;
  auto load8 = [&](int k, float (&v)[8]) {
    if constexpr (sizeof(T) == 2) {
      const uint4 u = *reinterpret_cast<const uint4*>(xr + k);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = unpack_bf16x2(w[i]);
        v[2 * i] = f.x; v[2 * i + 1] = f.y;
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(xr + k), b = *reinterpret_cast<const float4*>(xr + k + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
  };
  float amax = 0.f;
  for (int k = 8 * lane; k < K; k += 256) {
    float v[8];
    load8(k, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* qr = q + static_cast<int64_t>(row) * K;
  for (int k = 8 * lane; k < K; k += 256) {
    float v[8];
    load8(k, v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t c = __nv_cvt_float_to_fp8(__fdiv_rn(v[i], s), __NV_SATFINITE, __NV_E4M3);
      w[i >> 2] |= c << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(qr + k) = make_uint2(w[0], w[1]);
  }
  if (lane == 0) scale[row] = s;
}

// The same quantisation for bf16 rows read once: the row stays in registers
// between its maximum and its codes.  WPR warps per row (1 for K <= 2048, 8 for
// K <= 16384; their maxima meet in shared memory), 256 threads per block, each
// thread holding up to 8 chunks of 8 consecutive elements.
template <int WPR>
__global__ void __launch_bounds__(256) k_quant_rows_e4m3_reg(const bf16* __restrict__ x, int rows, int K,
                                                              uint8_t* __restrict__ q, float* __restrict__ scale) {
  constexpr int NV = 8, TPR = 32 * WPR, RPB = 8 / WPR;
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rib = warp / WPR, tir = (warp % WPR) * 32 + lane;   // row in block, thread in row
  const int row = blockIdx.x * RPB + rib;
  const bool live = row < rows;
  const bf16* xr = x + static_cast<int64_t>(live ? row : 0) * K;
  uint4 u[NV];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int k = (j * TPR + tir) * 8;
    u[j] = (live && k < K) ? *reinterpret_cast<const uint4*>(xr + k) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = unpack_bf16x2(w[i]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if constexpr (WPR > 1) {
    if (lane == 0) red[warp] = amax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < WPR; ++w) amax = fmaxf(amax, red[rib * WPR + w]);
  }
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* qr = q + static_cast<int64_t>(live ? row : 0) * K;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int k = (j * TPR + tir) * 8;
    if (!live || k >= K) continue;
    const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
    uint32_t c[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = unpack_bf16x2(w[i]);
      const uint32_t pair = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s)), __NV_SATFINITE, __NV_E4M3));   // f.x in the low byte
      c[i >> 1] |= pair << (16 * (i & 1));
    }
    *reinterpret_cast<uint2*>(qr + k) = make_uint2(c[0], c[1]);
  }
  if (live && tir == 0) scale[row] = s;
}

template <typename T>
wd_status quant_rows_e4m3(int rows, int K, const T* x, uint8_t* q, float* scale, cudaStream_t st) {
  if (rows <= 0 || K <= 0 || K % 8) { set_error("quant_rows: rows=%d, K=%d (K a multiple of 8)", rows, K); return WD_ERR_SHAPE; }
  Trace tr(KC_SMALL, st);
  if constexpr (std::is_same<T, bf16>::value) {
    if (K <= 2048) {          // one warp per row, 8 rows per block
      k_quant_rows_e4m3_reg<1><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(x, rows, K, q, scale);
      return launch_status("quant_rows_e4m3");
    }
    if (K <= 16384) {         // one block of 8 warps per row
      k_quant_rows_e4m3_reg<8><<<static_cast<unsigned>(rows), 256, 0, st>>>(x, rows, K, q, scale);
      return launch_status("quant_rows_e4m3");
    }
  }
  const int64_t threads = static_cast<int64_t>(rows) * 32;
  k_quant_rows_e4m3<T><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(x, rows, K, q, scale);
  return launch_status("quant_rows_e4m3");
}
template wd_status quant_rows_e4m3<bf16>(int, int, const bf16*, uint8_t*, float*, cudaStream_t);
template wd_status quant_rows_e4m3<float>(int, int, const float*, uint8_t*, float*, cudaStream_t);

}  // namespace wd
