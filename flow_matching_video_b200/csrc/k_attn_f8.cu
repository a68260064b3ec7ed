// k_attn_f8.cu — the FP8 self-attention of "Wan（通义万相）…" 5.3
// ("FlashAttention3 FP8": the Q/K inner product in INT8, O = P V in FP8,
// accumulation across key blocks in FP32) on the sm_100a tensor cores.
//
// Operands (k_attn8_prep, k_attn8_vt):
//   q8  int8, one scale per (token, head)        sq = amax / 127
//   k8  int8, one scale per (128-key block, head) sk = amax / 127
//   v8t e4m3, one scale per (channel, head, batch) sv = amax / 448, stored
//       transposed ([batch, heads, dh, Lkp]: keys contiguous) so that both
//       products read K-major operands
// Attention (k_attn_f8): per 128-key block, S = q8 k8^T in int32 by
// tcgen05.mma kind::i8 (exact: |S| <= 128 * 127^2 < 2^22), logits
// t = S sq sk log2(e) / sqrt(dh), the online softmax of the bf16 kernel (lazy
// reference max, threshold 8 in log2 units), p = 2^(t - m) <= 2^8 rounded to
// e4m3 into TMEM over the block's S columns (4 keys per 32-bit column), and
// O += P8 v8 by tcgen05.mma kind::f8f6f4 with P read from TMEM; the row sum l
// takes the unrounded p; out = O sv / l in bf16.
//
// CTA layout as in k_attn_tc's self-attention: two 128-row Q tiles of one
// (batch, head) ping-pong; warp 0 loads (TMA), warp 1 owns TMEM and issues the
// MMAs, warps 2..9 run the softmax (one thread per query row).
#include "wd_internal.cuh"

#include <cuda_fp8.h>

namespace wd {
namespace tc8 {

constexpr int BQ = 128, DH = 128, BK = 128, NQ = 2;
constexpr int TILE = 128 * 128;                 // one tile of 1-byte elements: 128 rows x 128 bytes
constexpr int RING = 8;                         // K8 / V8T tiles in flight (128 KB)
constexpr int PP = 2;                           // P of a block released to its P V in two parts
constexpr int THREADS = 64 + 32 * 4 * NQ;       // loader, MMA, four softmax warps per Q tile
constexpr int Q_OFF = 0, RING_OFF = NQ * TILE, BAR_OFF = RING_OFF + RING * TILE;
constexpr int SMEM = 1024 + BAR_OFF + 512;
constexpr float RESCALE_THRESHOLD = 8.0f;       // log2 units; p <= 2^8 stays below e4m3's 448
constexpr uint32_t MAGIC = 0x4B400000u;         // bits of 1.5 * 2^23: int32 s < 2^22 -> float 1.5 * 2^23 + s
constexpr float MAGIC_F = 12582912.f;

// TMEM (512 columns): tile t's S (int32) at 256 t, its O (fp32) at 256 t + 128;
// P8 overwrites the first 32 columns of S.
__host__ __device__ constexpr uint32_t s_col(int t) { return 256u * t; }
__host__ __device__ constexpr uint32_t o_col(int t) { return 256u * t + 128u; }

// Instruction descriptor of kind::i8: signed 8-bit A and B (format 1), int32
// accumulator (D format 2); the bit layout of the kind::f16 descriptor.
__host__ __device__ constexpr uint32_t idesc_s8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
constexpr uint32_t IDESC_S = idesc_s8(128, BK);
constexpr uint32_t IDESC_O = idesc_e4m3(128, DH, 0, 0);   // P (TMEM) x V^T (K-major)

enum : unsigned { SITE_Q = 0x301, SITE_KVF = 0x302, SITE_KVE = 0x303, SITE_S = 0x304, SITE_P = 0x305,
                  SITE_O = 0x306, SITE_DRAIN = 0x307 };

struct Params {
  int Lq, Lk, heads, nb;        // nb = ceil(Lk / 128)
  const float* sq;              // [batch, heads, Lq]
  const float* sk;              // [batch, heads, nb]
  const float* sv;              // [batch, heads * dh]
  bf16* o;
  int64_t o_rs;
  float scale_log2;             // log2(e) / sqrt(dh)
};

// D[tmem] (+)= A[smem] * B[smem]^T, signed int8 operands, shape M x N x 32.
__device__ __forceinline__ void umma_ss_i8_lh(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                              uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], da, db, %5, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, e4m3 operands (A: 4 elements per 32-bit column), shape M x N x 32.
__device__ __forceinline__ void umma_ts_f8_lh(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe for two lanes: the packed form of k_attn_tc's exp2_fma2
// (range reduction by the 1.5 * 2^23 rounding trick, this library's fitted
// degree-3 polynomial on [-1/2, 1/2], exponent added to the bits).
__device__ __forceinline__ float2 exp2_fma2_f8(float2 x) {
  x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 magic = make_float2(MAGIC_F, MAGIC_F);
  const float2 t = fadd2(x, magic);
  const float2 f = fsub2(x, fsub2(t, magic));
  const float2 c3 = make_float2(0.0551716648f, 0.0551716648f), c2 = make_float2(0.2426111251f, 0.2426111251f);
  const float2 c1 = make_float2(0.6932609677f, 0.6932609677f), c0 = make_float2(0.9999280572f, 0.9999280572f);
  const float2 q = ffma2(ffma2(ffma2(c3, f, c2), f, c1), f, c0);
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// Of every 8 exponentials, this many on the FMA pipe (even values: keys go in
// pairs).  0: all on MUFU.  The softmax here is issue-bound (int32 -> float
// conversion and e4m3 packing come on top of the bf16 kernel's work), so the
// polynomial's extra instructions cost more than the MUFU time they free
// (B200, 480p block, batch 2: 10.06 ms with 0, 11.38 ms with 2, 12.11 with 4).
#ifndef WD_F8_EXP2_EMU_PER8
#define WD_F8_EXP2_EMU_PER8 0
#endif
// int32 S -> float (exact either way): 1 uses the conversion instruction; 0 adds
// the bits of 1.5 * 2^23 and subtracts 1.5 * 2^23 as a float.  The conversion
// was faster (B200, 480p block, batch 2: 10.37 against 10.96 ms).
#ifndef WD_F8_CVT
#define WD_F8_CVT 1
#endif
constexpr float S_OFF = WD_F8_CVT ? 0.f : MAGIC_F;   // the offset the float values of S carry

// e4m3 codes of two floats, x in the low byte (round to nearest even, saturating)
__device__ __forceinline__ uint32_t e4m3x2(float x, float y) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(x, y), __NV_SATFINITE, __NV_E4M3));
}

__global__ void __launch_bounds__(THREADS, 1)
k_attn_f8(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* q_full = bars;                 // 1
  uint64_t* kv_full = bars + 1;            // RING
  uint64_t* kv_empty = kv_full + RING;     // RING
  uint64_t* s_full = kv_empty + RING;      // NQ
  uint64_t* p_full = s_full + NQ;          // NQ: all of P written
  uint64_t* p_part = p_full + NQ;          // NQ: the first half of P written
  uint64_t* o_done = p_part + NQ;          // NQ
  uint64_t* tdone = o_done + NQ;           // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int l0 = qb * BQ * NQ;
  const int NB = p.nb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < RING; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);
      mbar_init(&p_part[t], 4);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(tdone, 1);
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loader
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0, last_par = 0;
      mbar_arrive_expect_tx(q_full, NQ * TILE);
      for (int t = 0; t < NQ; ++t) tma_load_3d(smem + Q_OFF + t * TILE, &tmQ, h * DH, l0 + t * BQ, b, q_full);
      for (int n = 0; n < NB && ok; ++n) {
        for (int kv = 0; kv < 2; ++kv) {
          const int seq = 2 * n + kv, slot = seq % RING;
          const uint32_t ph = (seq / RING) & 1u;
          if (!mbar_wait(&kv_empty[slot], ph ^ 1u, SITE_KVE)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[slot], TILE);
          if (kv == 0)   // K8 rows n*128.. of head h: x = head column, y = key
            tma_load_3d(smem + RING_OFF + slot * TILE, &tmK, h * DH, n * BK, b, &kv_full[slot]);
          else           // V8T rows h*128.. (channels), x = key
            tma_load_3d(smem + RING_OFF + slot * TILE, &tmV, n * BK, h * DH, b, &kv_full[slot]);
          issued |= 1u << slot;
          last_par = (last_par & ~(1u << slot)) | (ph << slot);
        }
      }
      mbar_wait(q_full, 0, SITE_DRAIN);
      for (int s = 0; s < RING; ++s)
        if (issued & (1u << s)) mbar_wait(&kv_full[s], (last_par >> s) & 1u, SITE_DRAIN);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, SITE_Q);
      tc_fence_after();
      // K-major 128-byte rows, 128-byte swizzle, 8-row groups 1024 bytes apart;
      // a k-step of 32 one-byte elements advances the start address by 32 bytes.
      const uint64_t dq = sdesc_sw128(smem_u32(smem + Q_OFF), 16, 1024);
      const uint64_t dr = sdesc_sw128(smem_u32(smem + RING_OFF), 16, 1024);
      const uint32_t q_lo = static_cast<uint32_t>(dq), r_lo = static_cast<uint32_t>(dr);
      const uint32_t d_hi = static_cast<uint32_t>(dq >> 32);
      auto issue_s = [&](int t, int n) {
        const int kslot = (2 * n) % RING;
        const uint32_t qa = q_lo + t * (TILE >> 4), kb = r_lo + kslot * (TILE >> 4);
#pragma unroll
        for (int kk = 0; kk < DH / 32; ++kk)
          umma_ss_i8_lh(tmem + s_col(t), qa + kk * 2, d_hi, kb + kk * 2, d_hi, IDESC_S, kk ? 1u : 0u);
        umma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int n) -> bool {
        const int vseq = 2 * n + 1, vslot = vseq % RING;
        const uint32_t vb = r_lo + vslot * (TILE >> 4);
#pragma unroll
        for (int part = 0; part < PP; ++part) {
          if (!mbar_wait(part == 0 ? &p_part[t] : &p_full[t], n & 1u, SITE_P)) return false;
          if (part == 0 && t == 0 && !mbar_wait(&kv_full[vslot], (vseq / RING) & 1u, SITE_KVF)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = part * 2; kk < part * 2 + 2; ++kk)   // 32 keys: 8 TMEM columns of P, 32 bytes of V^T rows
            umma_ts_f8_lh(tmem + o_col(t), tmem + s_col(t) + kk * 8, vb + kk * 2, d_hi, IDESC_O, (n | kk) ? 1u : 0u);
        }
        if (t == NQ - 1) umma_commit(&kv_empty[vslot]);
        return true;
      };
      for (int n = 0; n < NB && ok; ++n) {
        for (int t = 0; t < NQ && ok; ++t) {
          // P V of the previous block first: it needs only that P and V tile
          if (n > 0 && !issue_pv(t, n - 1)) { ok = false; break; }
          if (t == 0) {
            const int kseq = 2 * n;
            if (!mbar_wait(&kv_full[kseq % RING], (kseq / RING) & 1u, SITE_KVF)) { ok = false; break; }
            tc_fence_after();
          }
          issue_s(t, n);
        }
        if (ok) umma_commit(&kv_empty[(2 * n) % RING]);
      }
      for (int t = 0; t < NQ && ok; ++t) {
        if (!issue_pv(t, NB - 1)) { ok = false; break; }
        umma_commit(&o_done[t]);
      }
      umma_commit(tdone);
      mbar_wait(tdone, 0, SITE_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int sw = warp - 2;
    const int t = sw >> 2;                 // Q tile
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;     // query row within the tile
    const int row = l0 + t * BQ + r;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + s_col(t);
    const int64_t bh = static_cast<int64_t>(b) * p.heads + h;
    const float cq = (row < p.Lq ? p.sq[bh * p.Lq + row] : 1.f) * p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < NB; ++n) {
      const float cl = cq * p.sk[bh * NB + n];            // log2 units per unit of the int32 product
      if (!mbar_wait_warp(&s_full[t], n & 1u, SITE_S)) { ok = false; break; }
      tc_fence_after();
      const int valid = p.Lk - n * BK;
      uint32_t a[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, a[c]);
      tmem_wait_ld();
      // int32 -> float: 1.5 * 2^23 + s as float bits, or s itself (exact either way); masked keys -> -inf
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int k = 0; k < 32; ++k)
          a[c][k] = WD_F8_CVT ? __float_as_uint(__int2float_rn(static_cast<int>(a[c][k]))) : a[c][k] + MAGIC;
      if (valid < BK) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (c * 32 + k >= valid) a[c][k] = __float_as_uint(-INFINITY);
      }
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 4; c += 2)
#pragma unroll
        for (int k = 0; k < 32; k += 2)
          m4[(k >> 1) & 3] = fmax3(m4[(k >> 1) & 3],
                                   fmax3(__uint_as_float(a[c][k]), __uint_as_float(a[c][k + 1]),
                                         __uint_as_float(a[c + 1][k])),
                                   __uint_as_float(a[c + 1][k + 1]));
      const float mx = (fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) - S_OFF) * cl;
      const bool grow = mx > m + RESCALE_THRESHOLD;
      const float m_new = grow ? mx : m;
      const float alpha = grow ? ex2f(m - m_new) : 1.f;
      m = m_new;
      // O *= alpha for rows whose reference moved, before this block's P V
      // (P V of the previous block has completed: its commit precedes S's)
      if (__any_sync(0xffffffffu, grow) && n > 0) {
        const uint32_t o_addr = tmem + lane_base + o_col(t);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(o_addr + c * 32, o);
        }
        tmem_wait_st();
      }
      // p = 2^(s cl - m) (s exact: the magic offset is subtracted before the scale);
      // 32 keys -> 8 columns of e4m3 codes over this row's S columns 8c..8c+7
      float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 mg2 = make_float2(MAGIC_F, MAGIC_F), cl2 = make_float2(cl, cl), nm2 = make_float2(-m, -m);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          float e[4];
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            float2 x = make_float2(__uint_as_float(a[c][k + j]), __uint_as_float(a[c][k + j + 1]));
            if (!WD_F8_CVT) x = fsub2(x, mg2);
            const float2 arg = ffma2(x, cl2, nm2);
            if (((k + j) & 7) >= 8 - WD_F8_EXP2_EMU_PER8) {
              const float2 y = exp2_fma2_f8(arg);
              e[j] = y.x;
              e[j + 1] = y.y;
            } else {
              e[j] = ex2f(arg.x);
              e[j + 1] = ex2f(arg.y);
            }
            rs4[((k + j) >> 1) & 3] = fadd2(rs4[((k + j) >> 1) & 3], make_float2(e[j], e[j + 1]));
          }
          pk[k >> 2] = e4m3x2(e[0], e[1]) | (e4m3x2(e[2], e[3]) << 16);   // keys k..k+3, low byte first
        }
        tmem_st8(s_addr + c * 8, pk);
        if (c == 1) {   // keys 0..63 written: release the first half of P V
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_part[t]);
        }
      }
      tmem_wait_st();
      const float2 rs2 = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
      l = l * alpha + (rs2.x + rs2.y);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------- epilogue: out = O sv / l
    if (ok && mbar_wait_warp(&o_done[t], 0, SITE_O)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const float* sv = p.sv + static_cast<int64_t>(b) * p.heads * DH + h * DH;
      bf16* dst = p.o + (static_cast<int64_t>(b) * p.Lq + row) * p.o_rs + h * DH;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + o_col(t) + c * 32, o);
        tmem_wait_ld();
        if (row < p.Lq) {
          float v[32];
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const float4 s4 = __ldg(reinterpret_cast<const float4*>(sv + c * 32 + k));
            v[k] = __uint_as_float(o[k]) * s4.x * inv;
            v[k + 1] = __uint_as_float(o[k + 1]) * s4.y * inv;
            v[k + 2] = __uint_as_float(o[k + 2]) * s4.z * inv;
            v[k + 3] = __uint_as_float(o[k + 3]) * s4.w * inv;
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                               pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ operand preparation
// One CTA per (128-row tile, head, batch), 8 warps of 16 rows, 4 channels per
// lane.  Q rows (tile rows < Lq): int8 with one scale per row.  K rows (tile
// rows < Lk): int8 with one scale for the tile (the attention's key block).
// V rows: the tile's per-channel |v| maxima folded into v_amax (float bits,
// atomicMax: the values are non-negative, so the integer order is the float order).
struct PrepArgs {
  const bf16* q; int64_t q_rs;            // q row (b, l): q + (b * Lq + l) * q_rs + h * 128
  const bf16* k; const bf16* v; int64_t kv_rs;
  int Lq, Lk, heads, nb;
  int8_t* q8; float* sq;                  // [batch, Lq, heads*128], [batch, heads, Lq]
  int8_t* k8; float* sk;                  // [batch, Lk, heads*128], [batch, heads, nb]
  unsigned* v_amax;                       // [batch, heads*128], zeroed before the launch
};

// Four int8 codes round-half-even(x / s), x[0] in the low byte.  The rounding to
// an integer adds 1.5 * 2^23 (exact round-to-nearest-even for |y| < 2^22; here
// |x / s| <= 127), which keeps it off the conversion unit.
__device__ __forceinline__ uint32_t i8x4(const float (&x)[4], float s) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float y = __fdiv_rn(x[j], s);
    const int c = max(-127, min(127, __float_as_int(__fadd_rn(y, MAGIC_F)) - static_cast<int>(MAGIC)));
    w |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * j);
  }
  return w;
}

__global__ void __launch_bounds__(256, 2) k_attn8_prep(PrepArgs a) {
  __shared__ float red[8][128];
  __shared__ float kred[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int D = a.heads * 128, col = h * 128 + lane * 4;
  const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
  const int r0 = tile * 128 + warp * 16;   // this warp's first row
  // each phase issues all its loads of the warp's 16 rows before any arithmetic (rows past the end read as 0)
  uint2 uq[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int l = r0 + i;
    uq[i] = l < a.Lq ? *reinterpret_cast<const uint2*>(a.q + (static_cast<int64_t>(b) * a.Lq + l) * a.q_rs + col)
                     : make_uint2(0u, 0u);
  }
  auto unpack = [](uint2 u, float (&x)[4]) {
    const float2 p0 = unpack_bf16x2(u.x), p1 = unpack_bf16x2(u.y);
    x[0] = p0.x; x[1] = p0.y; x[2] = p1.x; x[3] = p1.y;
  };
  // ---- Q: one scale per row
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int l = r0 + i;
    float x[4];
    unpack(uq[i], x);
    float am = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    const float s = am > 0.f ? __fdiv_rn(am, 127.f) : 1.f;
    if (l < a.Lq) {
      *reinterpret_cast<uint32_t*>(a.q8 + (static_cast<int64_t>(b) * a.Lq + l) * D + col) = i8x4(x, s);
      if (lane == 0) a.sq[bh * a.Lq + l] = s;
    }
  }
  if (tile * 128 >= a.Lk) return;                        // CTA-uniform: no keys in this tile
  // ---- K (one scale for the tile's 128 keys) and V (per-channel maxima over the tile)
  uint2 uk[16], uv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int l = r0 + i;
    const int64_t off = (static_cast<int64_t>(b) * a.Lk + l) * a.kv_rs + col;
    uk[i] = l < a.Lk ? *reinterpret_cast<const uint2*>(a.k + off) : make_uint2(0u, 0u);
    uv[i] = l < a.Lk ? *reinterpret_cast<const uint2*>(a.v + off) : make_uint2(0u, 0u);
  }
  float km = 0.f, vm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x[4], y[4];
    unpack(uk[i], x);
    unpack(uv[i], y);
#pragma unroll
    for (int j = 0; j < 4; ++j) { km = fmaxf(km, fabsf(x[j])); vm[j] = fmaxf(vm[j], fabsf(y[j])); }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
#pragma unroll
  for (int j = 0; j < 4; ++j) red[warp][lane * 4 + j] = vm[j];
  if (lane == 0) kred[warp] = km;
  __syncthreads();
  if (threadIdx.x < 128) {
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w][threadIdx.x]);
    atomicMax(&a.v_amax[static_cast<int64_t>(b) * D + h * 128 + threadIdx.x], __float_as_uint(m));
  }
  float km_all = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) km_all = fmaxf(km_all, kred[w]);
  const float s = km_all > 0.f ? __fdiv_rn(km_all, 127.f) : 1.f;
  if (threadIdx.x == 0) a.sk[bh * a.nb + tile] = s;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int l = r0 + i;
    float x[4];
    unpack(uk[i], x);
    if (l < a.Lk) *reinterpret_cast<uint32_t*>(a.k8 + (static_cast<int64_t>(b) * a.Lk + l) * D + col) = i8x4(x, s);
  }
}

// V -> e4m3 per channel, transposed: one CTA per (128-key tile, head, batch).
// sv = amax / 448 (1 for an all-zero channel); v8t[b, h, d, key] = e4m3(v / sv),
// keys Lk..Lkp of the last tile written as 0.  The tile-0 CTA writes sv.
struct VtArgs {
  const bf16* v; int64_t kv_rs;
  int Lk, heads;
  int64_t lkp;
  const unsigned* v_amax;
  uint8_t* v8t;                           // [batch, heads, 128, lkp]
  float* sv;                              // [batch, heads*128]
};

__global__ void __launch_bounds__(256) k_attn8_vt(VtArgs a) {
  __shared__ __align__(16) uint8_t tile_t[128][128 + 16];   // [channel][key]; 16 bytes of padding per row
  __shared__ float sc[128];
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int D = a.heads * 128;
  if (threadIdx.x < 128) {
    const float am = __uint_as_float(a.v_amax[static_cast<int64_t>(b) * D + h * 128 + threadIdx.x]);
    const float s = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
    sc[threadIdx.x] = s;
    if (tile == 0) a.sv[static_cast<int64_t>(b) * D + h * 128 + threadIdx.x] = s;
  }
  __syncthreads();
  // thread -> keys 4 kq .. 4 kq + 3, channels 16 cg .. 16 cg + 15 (one 32-byte sector of each row):
  // all loads first, then one 32-bit word of four keys' codes per channel into the transposed tile
  const int kq = threadIdx.x & 31, cg = threadIdx.x >> 5;
  uint4 u[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int l = tile * 128 + 4 * kq + i;
    const bf16* src = a.v + (static_cast<int64_t>(b) * a.Lk + l) * a.kv_rs + h * 128 + 16 * cg;
    u[i][0] = l < a.Lk ? *reinterpret_cast<const uint4*>(src) : make_uint4(0u, 0u, 0u, 0u);   // keys past the end: 0
    u[i][1] = l < a.Lk ? *reinterpret_cast<const uint4*>(src + 8) : make_uint4(0u, 0u, 0u, 0u);
  }
  auto val = [&](int i, int c) {   // key 4 kq + i, channel 16 cg + c
    const uint4 q = u[i][c >> 3];
    const uint32_t w = ((c & 7) >> 1) == 0 ? q.x : ((c & 7) >> 1) == 1 ? q.y : ((c & 7) >> 1) == 2 ? q.z : q.w;
    const float2 f = unpack_bf16x2(w);
    return (c & 1) ? f.y : f.x;
  };
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float s = sc[16 * cg + c];
    const uint32_t lo = e4m3x2(__fdiv_rn(val(0, c), s), __fdiv_rn(val(1, c), s));
    const uint32_t hi = e4m3x2(__fdiv_rn(val(2, c), s), __fdiv_rn(val(3, c), s));
    *reinterpret_cast<uint32_t*>(&tile_t[16 * cg + c][4 * kq]) = lo | (hi << 16);
  }
  __syncthreads();
  // rows of 128 keys (the last tile: up to lkp, a multiple of 16), 16 bytes per store
  const int64_t rem = a.lkp - static_cast<int64_t>(tile) * 128;
  const int64_t kmax = rem < 128 ? rem : 128;
  uint8_t* dst = a.v8t + (static_cast<int64_t>(b) * a.heads + h) * 128 * a.lkp + static_cast<int64_t>(tile) * 128;
  for (int i = threadIdx.x; i < 128 * 8; i += 256) {
    const int d = i >> 3, seg = i & 7;
    if (seg * 16 < kmax)
      *reinterpret_cast<uint4*>(dst + d * a.lkp + seg * 16) = *reinterpret_cast<const uint4*>(&tile_t[d][seg * 16]);
  }
}

}  // namespace tc8

// ------------------------------------------------------------------ host side
// Byte offsets of the FP8 attention's operands in one buffer (256-byte aligned).
wd_status attn_fp8_layout(int batch, int64_t Lq, int64_t Lk, int heads, int dh, wd_attn_fp8_layout* L) {
  if (dh != 128) { set_error("FP8 attention: head dim %d (supported: 128)", dh); return WD_ERR_UNSUPPORTED; }
  if (batch < 1 || Lq < 1 || Lk < 1 || heads < 1) { set_error("FP8 attention: empty shape"); return WD_ERR_SHAPE; }
  if (Lq > (1 << 30) || Lk > (1 << 30)) { set_error("FP8 attention: sequence too long"); return WD_ERR_SHAPE; }
  const int64_t D = static_cast<int64_t>(heads) * dh, nb = (Lk + 127) / 128;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t o = 0;
  L->lkp = (Lk + 15) / 16 * 16;
  L->q8 = o;     o = al(o + static_cast<size_t>(batch * Lq * D));
  L->sq = o;     o = al(o + sizeof(float) * static_cast<size_t>(batch * heads * Lq));
  L->k8 = o;     o = al(o + static_cast<size_t>(batch * Lk * D));
  L->sk = o;     o = al(o + sizeof(float) * static_cast<size_t>(batch * heads * nb));
  L->v8t = o;    o = al(o + static_cast<size_t>(batch * D * L->lkp));
  L->sv = o;     o = al(o + sizeof(float) * static_cast<size_t>(batch * D));
  L->v_amax = o; o = al(o + sizeof(unsigned) * static_cast<size_t>(batch * D));
  L->bytes = o;
  return WD_OK;
}

wd_status attn_fp8_quantize(int batch, int Lq, int Lk, int heads, const bf16* q, int64_t q_rs, const bf16* k,
                            const bf16* v, int64_t kv_rs, void* buf, const wd_attn_fp8_layout& L, cudaStream_t st) {
  uint8_t* base = static_cast<uint8_t*>(buf);
  const int64_t D = static_cast<int64_t>(heads) * 128;
  const int nb = (Lk + 127) / 128;
  auto al8 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 7u) == 0; };
  auto al16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
  if (!al8(q) || !al8(k) || !al16(v) || (q_rs % 8) || (kv_rs % 8) || !al16(buf)) {
    set_error("FP8 attention: q, k 8-byte and v, buffer 16-byte aligned, row strides multiples of 8");
    return WD_ERR_ALIGN;
  }
  if (cudaMemsetAsync(base + L.v_amax, 0, sizeof(unsigned) * batch * D, st) != cudaSuccess)
    return launch_status("attn_fp8 memset");
  tc8::PrepArgs a{};
  a.q = q; a.q_rs = q_rs; a.k = k; a.v = v; a.kv_rs = kv_rs;
  a.Lq = Lq; a.Lk = Lk; a.heads = heads; a.nb = nb;
  a.q8 = reinterpret_cast<int8_t*>(base + L.q8); a.sq = reinterpret_cast<float*>(base + L.sq);
  a.k8 = reinterpret_cast<int8_t*>(base + L.k8); a.sk = reinterpret_cast<float*>(base + L.sk);
  a.v_amax = reinterpret_cast<unsigned*>(base + L.v_amax);
  {
    const int tiles = (max(Lq, Lk) + 127) / 128;
    Trace tr(KC_SMALL, st);
    tc8::k_attn8_prep<<<dim3(tiles, heads, batch), 256, 0, st>>>(a);
  }
  WD_TRY(launch_status("attn8_prep"));
  tc8::VtArgs vt{};
  vt.v = v; vt.kv_rs = kv_rs; vt.Lk = Lk; vt.heads = heads; vt.lkp = L.lkp;
  vt.v_amax = reinterpret_cast<const unsigned*>(base + L.v_amax);
  vt.v8t = base + L.v8t;
  vt.sv = reinterpret_cast<float*>(base + L.sv);
  {
    Trace tr(KC_SMALL, st);
    tc8::k_attn8_vt<<<dim3(nb, heads, batch), 256, 0, st>>>(vt);
  }
  return launch_status("attn8_vt");
}

// 3D tensor map of one-byte elements: [batches, rows, cols] (cols contiguous,
// row stride rs bytes, batch stride bs bytes), box 128 x 128 x 1, 128-byte swizzle.
static wd_status make_tmap_u8(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t batches,
                              int64_t rs, int64_t bs) {
  auto fn = encode_fn();
  if (!fn) { set_error("cuTensorMapEncodeTiled unavailable"); return WD_ERR_CUDA; }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batches)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(rs), static_cast<cuuint64_t>(bs)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { set_error("cuTensorMapEncodeTiled (u8) failed (%d)", static_cast<int>(r)); return WD_ERR_CUDA; }
  return WD_OK;
}

wd_status attn_fp8(int batch, int Lq, int Lk, int heads, const void* buf, const wd_attn_fp8_layout& L, bf16* o,
                   int64_t o_rs, cudaStream_t st) {
  const uint8_t* base = static_cast<const uint8_t*>(buf);
  const int64_t D = static_cast<int64_t>(heads) * 128;
  if ((reinterpret_cast<uintptr_t>(buf) & 255u) || (reinterpret_cast<uintptr_t>(o) & 15u) || (o_rs % 8)) {
    set_error("FP8 attention: buffer 256-byte and output 16-byte aligned, output row stride a multiple of 8");
    return WD_ERR_ALIGN;
  }
  CUtensorMap tq, tk, tv;
  WD_TRY(make_tmap_u8(&tq, base + L.q8, D, Lq, batch, D, D * Lq));
  WD_TRY(make_tmap_u8(&tk, base + L.k8, D, Lk, batch, D, D * Lk));
  WD_TRY(make_tmap_u8(&tv, base + L.v8t, L.lkp, D, batch, L.lkp, D * L.lkp));
  tc8::Params p{};
  p.Lq = Lq; p.Lk = Lk; p.heads = heads; p.nb = (Lk + 127) / 128;
  p.sq = reinterpret_cast<const float*>(base + L.sq);
  p.sk = reinterpret_cast<const float*>(base + L.sk);
  p.sv = reinterpret_cast<const float*>(base + L.sv);
  p.o = o; p.o_rs = o_rs;
  p.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  static bool attr[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 15]) {
    cudaFuncSetAttribute(tc8::k_attn_f8, cudaFuncAttributeMaxDynamicSharedMemorySize, tc8::SMEM);
    attr[dev & 15] = true;
  }
  dim3 grid((Lq + tc8::BQ * tc8::NQ - 1) / (tc8::BQ * tc8::NQ), heads, batch);
  Trace tr(KC_ATTN_SELF, st);
  tc8::k_attn_f8<<<grid, tc8::THREADS, tc8::SMEM, st>>>(tq, tk, tv, p);
  return launch_status("attention_fp8");
}

}  // namespace wd
