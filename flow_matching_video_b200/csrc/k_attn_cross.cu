// k_attn_cross.cu — the decoupled image/text cross-attention of the DiT block
// ("图解 Wan2.1 I2V" 5.4: two softmaxes, over the 257 image keys and over the
// 512 text keys, summed after normalisation) with the two segments computed
// side by side.
//
// The arithmetic per segment is that of k_attn_tc (S = Q K^T into TMEM, the
// online softmax with the lazy reference max, P in TMEM for the P V TS-MMA).
// The two segments are independent softmaxes, so they run as two chains at
// once, each with its own softmax warpgroup, S buffer and O accumulator:
// while one chain's warps run their softmax, the tensor cores run the other
// chain's MMAs, and every SM sub-partition holds two softmax warps.  (Walking
// the segments one after the other left one softmax warp per sub-partition
// with nothing to hide its latency behind.)
//
// CTA = one 128-row Q tile of one (batch, head):
//   warp 0      TMA: lane 0 loads Q and the image chain's K/V, lane 1 the text
//               chain's, each through its own 3-slot ring
//   warp 1      TMEM owner + MMA issuer for both chains
//   warps 2..5  softmax of the image keys (chain 0)
//   warps 6..9  softmax of the text keys (chain 1); they also write the output
//               O_text / l_text + O_image / l_image once both chains are done
// TMEM (512 columns): S of chain 0 at 0, O of chain 0 at 128, O of chain 1 at
// 256, S of chain 1 at 384.
#include "wd_internal.cuh"

namespace wd {
namespace tcx {

constexpr int BQ = 128, DH = 128, BK = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;     // a Q, K or V tile of 2-byte elements: two 64-column halves
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int RING = 3;                       // K/V tiles in flight per chain
constexpr int THREADS = 64 + 256;
constexpr int Q_OFF = 0, RING_OFF = TILE_BYTES, ST_OFF = RING_OFF + 2 * RING * TILE_BYTES;
constexpr int BAR_OFF = ST_OFF + 128 * 4;     // after the image chain's row sums
constexpr int SMEM = 1024 + BAR_OFF + 512;
static_assert(SMEM <= 232448, "shared memory budget of one CTA exceeded");
constexpr float RESCALE_THRESHOLD = 8.0f;     // log2 units

__host__ __device__ constexpr uint32_t s_col(int c) { return c ? 384u : 0u; }
__host__ __device__ constexpr uint32_t o_col(int c) { return 128u + 128u * c; }

enum : unsigned { SITE_Q = 0x401, SITE_KVF = 0x402, SITE_KVE = 0x403, SITE_S = 0x404, SITE_P = 0x405,
                  SITE_O = 0x406, SITE_DRAIN = 0x407, SITE_ST = 0x408 };

struct Seg {
  int n;        // keys
  int shared;   // keys shared by the batch (tensor map batch extent 1)
};

struct Params {
  int Lq;
  Seg seg[2];
  bf16* o;
  int64_t o_rs;
  float scale_log2;
};

template <typename TI>
__global__ void __launch_bounds__(THREADS, 1)
k_attn_cross(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK0,
             const __grid_constant__ CUtensorMap tmV0, const __grid_constant__ CUtensorMap tmK1,
             const __grid_constant__ CUtensorMap tmV1, const Params p) {
  using C = tca::Cfg<1, 2, TI, 128>;   // the operand forms and instruction descriptors of k_attn_tc
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* q_full = bars;                   // 1
  uint64_t* kv_full = q_full + 1;            // [2][RING]
  uint64_t* kv_empty = kv_full + 2 * RING;   // [2][RING]
  uint64_t* s_full = kv_empty + 2 * RING;    // [2]
  uint64_t* p_part = s_full + 2;             // [2]: keys 0..63 of the chain's block written as P
  uint64_t* p_full = p_part + 2;             // [2]
  uint64_t* o_done = p_full + 2;             // 1: every P V completed
  uint64_t* st_full = o_done + 1;            // 1: the image chain's row sums written
  uint64_t* tdone = st_full + 1;             // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tdone + 1);
  float* st = reinterpret_cast<float*>(smem + ST_OFF);   // [128]: l of the image chain per row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  int nb[2];
  nb[0] = (p.seg[0].n + BK - 1) / BK;
  nb[1] = (p.seg[1].n + BK - 1) / BK;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2 * RING; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&s_full[c], 1);
      mbar_init(&p_part[c], 4);
      mbar_init(&p_full[c], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(st_full, 4);
    mbar_init(tdone, 1);
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA: lane c loads chain c
    if (lane < 2) {
      const int c = lane;
      const CUtensorMap* tk = c ? &tmK1 : &tmK0;
      const CUtensorMap* tv = c ? &tmV1 : &tmV0;
      const int bb = p.seg[c].shared ? 0 : b;
      uint64_t* full = kv_full + c * RING;
      uint64_t* empty = kv_empty + c * RING;
      uint8_t* ring = smem + RING_OFF + c * RING * TILE_BYTES;
      if (c == 0) {
        mbar_arrive_expect_tx(q_full, TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + Q_OFF + hf * HALF_BYTES, &tmQ, h * DH + hf * 64, qb * BQ, b, q_full);
      }
      bool ok = true;
      uint32_t issued = 0, last_par = 0;
      for (int n = 0; n < nb[c] && ok; ++n) {
        for (int kv = 0; kv < 2; ++kv) {
          const int seq = 2 * n + kv, slot = seq % RING;
          const uint32_t ph = (seq / RING) & 1u;
          if (!mbar_wait(&empty[slot], ph ^ 1u, SITE_KVE)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[slot], TILE_BYTES);
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(ring + slot * TILE_BYTES + hf * HALF_BYTES, kv ? tv : tk, h * DH + hf * 64, n * BK, bb,
                        &full[slot]);
          issued |= 1u << slot;
          last_par = (last_par & ~(1u << slot)) | (ph << slot);
        }
      }
      // every copy this lane issued lands before the CTA can exit
      if (c == 0) mbar_wait(q_full, 0, SITE_DRAIN);
      for (int s = 0; s < RING; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1u, SITE_DRAIN);
    }
    __syncwarp();
  }
  else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, SITE_Q);
      tc_fence_after();
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + Q_OFF), 16, 1024);
      const uint32_t q_lo = static_cast<uint32_t>(dq0), s_hi = static_cast<uint32_t>(dq0 >> 32);
      uint32_t k_lo[2], v_lo[2], v_hi = 0;
      for (int c = 0; c < 2; ++c) {
        const uint32_t base = smem_u32(smem + RING_OFF + c * RING * TILE_BYTES);
        const uint64_t dk = sdesc_sw128(base, 16, 1024), dv = sdesc_sw128(base, HALF_BYTES, 1024);
        k_lo[c] = static_cast<uint32_t>(dk);
        v_lo[c] = static_cast<uint32_t>(dv);
        v_hi = static_cast<uint32_t>(dv >> 32);
      }
      // S_c = Q K^T of chain c's block n into its S buffer
      auto issue_s = [&](int c, int n) -> bool {
        const int seq = 2 * n, slot = seq % RING;
        if (!mbar_wait(&kv_full[c * RING + slot], (seq / RING) & 1u, SITE_KVF)) return false;
        tc_fence_after();
        const uint32_t d = tmem + s_col(c), kb = k_lo[c] + slot * (TILE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
          umma_ss_lh(d, q_lo + off, s_hi, kb + off, s_hi, C::IDESC_S, kk ? 1u : 0u);
        }
        umma_commit(&s_full[c]);
        umma_commit(&kv_empty[c * RING + slot]);   // K read
        return true;
      };
      // O_c (+)= P_c V of chain c's block n, in two halves of 64 keys as the softmax writes P
      auto issue_pv = [&](int c, int n) -> bool {
        const int seq = 2 * n + 1, slot = seq % RING;
        const uint32_t d = tmem + o_col(c), pa = tmem + s_col(c), vb = v_lo[c] + slot * (TILE_BYTES >> 4);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          if (!mbar_wait(part == 0 ? &p_part[c] : &p_full[c], n & 1u, SITE_P)) return false;
          if (part == 0 && !mbar_wait(&kv_full[c * RING + slot], (seq / RING) & 1u, SITE_KVF)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = part * 4; kk < part * 4 + 4; ++kk)   // 16 keys = 8 TMEM columns of P; 2048 bytes of V
            umma_ts_lh(d, pa + 8 * kk, vb + kk * (2048 >> 4), v_hi, C::IDESC_O, (n || kk) ? 1u : 0u);
        }
        umma_commit(&kv_empty[c * RING + slot]);   // V read
        return true;
      };
      // per block index, each chain's P V of the previous block, then its next S (S of a chain
      // is issued after its P V, so it never overwrites a P that P V has still to read)
      const int nmax = nb[0] > nb[1] ? nb[0] : nb[1];
      for (int n = 0; n <= nmax && ok; ++n)
        for (int c = 0; c < 2 && ok; ++c) {
          if (n >= 1 && n - 1 < nb[c]) ok = issue_pv(c, n - 1);
          if (ok && n < nb[c]) ok = issue_s(c, n);
        }
      if (ok) umma_commit(o_done);
      umma_commit(tdone);
      mbar_wait(tdone, 0, SITE_DRAIN);
    }
    __syncwarp();
  }
  else {
    // ------------------------------------------------------------ softmax warps of chain c
    const int c = (warp - 2) >> 2;
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;     // query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + s_col(c);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < nb[c]; ++n) {
      if (!mbar_wait_warp(&s_full[c], n & 1u, SITE_S)) { ok = false; break; }
      tc_fence_after();
      const int valid = p.seg[c].n - n * BK;   // keys of this block that exist
      uint32_t a[4][32];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) tmem_ld32(s_addr + k4 * 32, a[k4]);
      tmem_wait_ld();
      if (valid < BK) {
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k4 * 32 + k >= valid) a[k4][k] = __float_as_uint(-INFINITY);
      }
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int k4 = 0; k4 < 4; k4 += 2)
#pragma unroll
        for (int k = 0; k < 32; k += 2)
          m4[(k >> 1) & 3] = fmax3(m4[(k >> 1) & 3],
                                   fmax3(__uint_as_float(a[k4][k]), __uint_as_float(a[k4][k + 1]),
                                         __uint_as_float(a[k4 + 1][k])),
                                   __uint_as_float(a[k4 + 1][k + 1]));
      const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * p.scale_log2;
      // lazy rescale: the reference moves only when the block's maximum exceeds it by the threshold
      const bool grow = mx > m + RESCALE_THRESHOLD;
      const float m_new = grow ? mx : m;
      const float alpha = grow ? tca::ex2(m - m_new) : 1.f;
      m = m_new;
      if (__any_sync(0xffffffffu, grow) && n > 0) {
        // O_c *= alpha: the chain's previous P V has completed (its S commit came after it)
        const uint32_t o_addr = tmem + lane_base + o_col(c);
#pragma unroll 1
        for (int k4 = 0; k4 < 4; ++k4) {
          uint32_t o[32];
          tmem_ld32(o_addr + k4 * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(o_addr + k4 * 32, o);
        }
        tmem_wait_st();
      }
      // P = 2^(s scale - m) in the operand type over the chain's S columns (chunk q of 16 keys
      // -> 8 columns at 8q), released to P V in two halves
      float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-m, -m);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const int kk = (q & 1) * 16 + k;
          const float2 arg = ffma2(make_float2(__uint_as_float(a[q >> 1][kk]), __uint_as_float(a[q >> 1][kk + 1])),
                                   sc2, nm2);
          float e0, e1;
          if (WD_EXP2_PACKED && (k & 7) >= 8 - WD_EXP2_EMU_PER8 && ((k + 1) & 7) >= 8 - WD_EXP2_EMU_PER8) {
            const float2 e = tca::exp2_fma2(arg);
            e0 = e.x;
            e1 = e.y;
          } else {
            e0 = ((k & 7) >= 8 - WD_EXP2_EMU_PER8) ? tca::exp2_fma(arg.x) : tca::ex2(arg.x);
            e1 = (((k + 1) & 7) >= 8 - WD_EXP2_EMU_PER8) ? tca::exp2_fma(arg.y) : tca::ex2(arg.y);
          }
          rs4[(k >> 1) & 3] = fadd2(rs4[(k >> 1) & 3], make_float2(e0, e1));
          pk[k >> 1] = C::HALF ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
        }
        tmem_st8(s_addr + q * 8, pk);
        if (q == 3) {   // keys 0..63 written
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_part[c]);
        }
      }
      tmem_wait_st();
      const float2 rs = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
      l = l * alpha + (rs.x + rs.y);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[c]);
    }
    if (c == 0) {
      // the image chain's row sums for the text chain's warps, which write the output
      if (ok) {
        st[r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(st_full);
      }
    } else if (ok && mbar_wait_warp(st_full, 0, SITE_ST) && mbar_wait_warp(o_done, 0, SITE_O)) {
      // out = O_text / l_text + O_image / l_image, rounded to bf16
      tc_fence_after();
      const float inv1 = 1.f / l, inv0 = 1.f / st[r];
      const int row = qb * BQ + r;
      bf16* dst = p.o + (static_cast<int64_t>(b) * p.Lq + row) * p.o_rs + h * DH;
#pragma unroll 1
      for (int k4 = 0; k4 < 4; ++k4) {
        uint32_t o[32];
        float v[32];
        tmem_ld32(tmem + lane_base + o_col(1) + k4 * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(o[k]) * inv1;
        tmem_ld32(tmem + lane_base + o_col(0) + k4 * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] += __uint_as_float(o[k]) * inv0;
        if (row < p.Lq) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + k4 * 32);
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

}  // namespace tcx

// ------------------------------------------------------------------ host side
// Two key segments (k1/v1 and k2/v2), head dim 128: one CTA per 128-row Q tile.
template <typename TI>
wd_status attention_cross_tc(const AttnArgs<TI, bf16>& a, cudaStream_t st) {
  const int D = a.heads * a.dh;
  const CUtensorMapDataType ty =
      std::is_same<TI, f16>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tq, tk0, tv0, tk1, tv1;
  WD_TRY(make_tmap_3d(&tq, ty, a.q, D, a.Lq, a.batch, a.q_rs, a.q_rs * a.Lq));
  const int64_t b1 = a.kv1_bs ? a.batch : 1, b2 = a.kv2_bs ? a.batch : 1;
  WD_TRY(make_tmap_3d(&tk0, ty, a.k1, D, a.n1, b1, a.kv1_rs, a.kv1_bs));
  WD_TRY(make_tmap_3d(&tv0, ty, a.v1, D, a.n1, b1, a.kv1_rs, a.kv1_bs));
  WD_TRY(make_tmap_3d(&tk1, ty, a.k2, D, a.n2, b2, a.kv2_rs, a.kv2_bs));
  WD_TRY(make_tmap_3d(&tv1, ty, a.v2, D, a.n2, b2, a.kv2_rs, a.kv2_bs));
  tcx::Params p{};
  p.Lq = a.Lq;
  p.seg[0] = tcx::Seg{a.n1, a.kv1_bs == 0};
  p.seg[1] = tcx::Seg{a.n2, a.kv2_bs == 0};
  p.o = a.o;
  p.o_rs = a.o_rs;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.dh));
  static bool attr[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 15]) {
    cudaFuncSetAttribute(tcx::k_attn_cross<TI>, cudaFuncAttributeMaxDynamicSharedMemorySize, tcx::SMEM);
    attr[dev & 15] = true;
  }
  dim3 grid((a.Lq + tcx::BQ - 1) / tcx::BQ, a.heads, a.batch);
  Trace tr(a.cross ? KC_ATTN_CROSS : KC_ATTN_SELF, st);
  tcx::k_attn_cross<TI><<<grid, tcx::THREADS, tcx::SMEM, st>>>(tq, tk0, tv0, tk1, tv1, p);
  return launch_status("attention_cross_tc");
}
template wd_status attention_cross_tc<bf16>(const AttnArgs<bf16, bf16>&, cudaStream_t);
template wd_status attention_cross_tc<f16>(const AttnArgs<f16, bf16>&, cudaStream_t);

}  // namespace wd
