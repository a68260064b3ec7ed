// k_attn_cross.cu — the decoupled image/text cross-attention of the DiT block
// ("图解 Wan2.1 I2V" 5.4: two softmaxes over the 257 image keys and the 512 text
// keys, summed after normalisation) as a persistent tcgen05 kernel.
//
// The arithmetic is that of k_attn_tc's two-segment kernel (S = Q K^T into
// TMEM, the online softmax with the lazy reference max, P in TMEM for the
// P V TS-MMA, one O accumulator per segment).  What differs is the schedule:
// a CTA runs one 128-row Q tile at a time but loops over tiles, so
//   - the next tile's Q is loaded into the second of two Q slots while the
//     current tile computes;
//   - the double-buffered S schedule runs over one sequence of key blocks
//     across tiles: S of the next tile's first blocks is computed while the
//     current tile finishes;
//   - a separate epilogue warpgroup reads O, normalises, sums the segments and
//     stores, then hands O back to the next tile's first P V, while the
//     softmax warps go on with the next tile.
// With 7 short key blocks per tile, the per-tile prologue and epilogue were a
// large part of each CTA's time; here they overlap the tensor cores.
//
// Warps: 0 TMA loader, 1 TMEM owner + MMA issuer, 2..5 softmax (one thread per
// query row), 6..9 epilogue.  TMEM (512 columns): S buffers at 0 and 384, O of
// the image segment at 128, O of the text segment at 256.
#include "wd_internal.cuh"

namespace wd {
namespace tcx {

constexpr int BQ = 128, DH = 128, BK = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;     // a Q, K or V tile of 2-byte elements: two 64-column halves
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int RING = 4;                       // K/V tiles in flight
constexpr int THREADS = 64 + 128 + 128;
constexpr int Q_OFF = 0, RING_OFF = 2 * TILE_BYTES, ST_OFF = RING_OFF + RING * TILE_BYTES;
constexpr int BAR_OFF = ST_OFF + 2 * 128 * 4;   // after the row sums handed to the epilogue
constexpr int SMEM = 1024 + BAR_OFF + 512;
static_assert(SMEM <= 232448, "shared memory budget of one CTA exceeded");
constexpr float RESCALE_THRESHOLD = 8.0f;     // log2 units
constexpr int PP = 2;                         // P of a block released to its P V in two halves

__host__ __device__ constexpr uint32_t s_col(int g) { return (g & 1) ? 384u : 0u; }
__host__ __device__ constexpr uint32_t o_col(int seg) { return 128u + 128u * seg; }

enum : unsigned { SITE_Q = 0x401, SITE_KVF = 0x402, SITE_KVE = 0x403, SITE_S = 0x404, SITE_P = 0x405,
                  SITE_O = 0x406, SITE_DRAIN = 0x407, SITE_QE = 0x408, SITE_OF = 0x409, SITE_ST = 0x40A };

struct Seg {
  int n;        // keys
  int shared;   // keys shared by the batch (tensor map batch extent 1)
};

struct Params {
  int Lq, heads, batch;
  int nqb;      // Q tiles per (batch, head)
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
  using C = tca::Cfg<1, 2, TI, 128>;   // the two-segment kernel's operand forms and descriptors
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* q_full = bars;              // 2
  uint64_t* q_empty = q_full + 2;       // 2
  uint64_t* kv_full = q_empty + 2;      // RING
  uint64_t* kv_empty = kv_full + RING;  // RING
  uint64_t* s_full = kv_empty + RING;   // 2 (S buffers)
  uint64_t* p_full = s_full + 2;        // 2
  uint64_t* p_part = p_full + 2;        // 2
  uint64_t* pv_done = p_part + 2;       // 2
  uint64_t* o_done = pv_done + 2;       // 1: the tile's last P V completed
  uint64_t* o_free = o_done + 1;        // 1: the epilogue has read O
  uint64_t* st_full = o_free + 1;       // 1: the softmax warps have written the tile's row sums
  uint64_t* tdone = st_full + 1;        // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tdone + 1);
  float* st = reinterpret_cast<float*>(smem + ST_OFF);   // [2][128]: l of the text segment, l of the image segment

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk0 = p.seg[0].n, nk1 = p.seg[1].n;
  const int nb0 = (nk0 + BK - 1) / BK, nb1 = (nk1 + BK - 1) / BK;
  const int NB = nb0 + nb1;
  const int items = p.nqb * p.heads * p.batch;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int n_items = blockIdx.x < items ? (items - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto tile_of = [&](int li, int& qb, int& h, int& b) {
    const int it = blockIdx.x + li * gridDim.x;
    qb = it % p.nqb;
    h = (it / p.nqb) % p.heads;
    b = it / (p.nqb * p.heads);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_part[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    for (int s = 0; s < RING; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(o_done, 1);
    mbar_init(o_free, 4);
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
    // ------------------------------------------------------------ TMA loader
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0, last_par = 0;
      uint32_t q_issued = 0, q_par = 0;
      int g = 0;   // key block sequence number over all of this CTA's tiles
      for (int li = 0; li < n_items && ok; ++li) {
        int qb, h, b;
        tile_of(li, qb, h, b);
        const int qs = li & 1;
        const uint32_t qph = (li >> 1) & 1u;
        if (!mbar_wait(&q_empty[qs], qph ^ 1u, SITE_QE)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[qs], TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + Q_OFF + qs * TILE_BYTES + hf * HALF_BYTES, &tmQ, h * DH + hf * 64, qb * BQ, b,
                      &q_full[qs]);
        q_issued |= 1u << qs;
        q_par = (q_par & ~(1u << qs)) | (qph << qs);
        for (int n = 0; n < NB && ok; ++n, ++g) {
          const int sg = n < nb0 ? 0 : 1;
          const int j0 = (n - (sg ? nb0 : 0)) * BK;
          const CUtensorMap* tk = sg ? &tmK1 : &tmK0;
          const CUtensorMap* tv = sg ? &tmV1 : &tmV0;
          const int bb = p.seg[sg].shared ? 0 : b;
          for (int kv = 0; kv < 2; ++kv) {
            const int seq = 2 * g + kv, slot = seq % RING;
            const uint32_t ph = (seq / RING) & 1u;
            if (!mbar_wait(&kv_empty[slot], ph ^ 1u, SITE_KVE)) { ok = false; break; }
            mbar_arrive_expect_tx(&kv_full[slot], TILE_BYTES);
            for (int hf = 0; hf < 2; ++hf)
              tma_load_3d(smem + RING_OFF + slot * TILE_BYTES + hf * HALF_BYTES, kv ? tv : tk, h * DH + hf * 64, j0,
                          bb, &kv_full[slot]);
            issued |= 1u << slot;
            last_par = (last_par & ~(1u << slot)) | (ph << slot);
          }
        }
      }
      // every copy this thread issued lands before the CTA can exit
      for (int s = 0; s < 2; ++s)
        if (q_issued & (1u << s)) mbar_wait(&q_full[s], (q_par >> s) & 1u, SITE_DRAIN);
      for (int s = 0; s < RING; ++s)
        if (issued & (1u << s)) mbar_wait(&kv_full[s], (last_par >> s) & 1u, SITE_DRAIN);
    }
    __syncwarp();
  }
  else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + Q_OFF), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(smem + RING_OFF), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(smem + RING_OFF), HALF_BYTES, 1024);
      const uint32_t q_lo = static_cast<uint32_t>(dq0), k_lo = static_cast<uint32_t>(dk0);
      const uint32_t v_lo = static_cast<uint32_t>(dv0);
      const uint32_t s_hi = static_cast<uint32_t>(dq0 >> 32), v_hi = static_cast<uint32_t>(dv0 >> 32);
      const int G = n_items * NB;   // key blocks of all this CTA's tiles, in order
      // S of block g (tile g / NB, its block g % NB) into S buffer g & 1
      auto issue_s = [&](int g) -> bool {
        const int li = g / NB, n = g % NB, qs = li & 1;
        if (n == 0) {   // the tile's Q
          if (!mbar_wait(&q_full[qs], (li >> 1) & 1u, SITE_Q)) return false;
        }
        const int kseq = 2 * g, kslot = kseq % RING;
        if (!mbar_wait(&kv_full[kslot], (kseq / RING) & 1u, SITE_KVF)) return false;
        tc_fence_after();
        const uint32_t d = tmem + s_col(g);
        const uint32_t qa = q_lo + qs * (TILE_BYTES >> 4), kb = k_lo + kslot * (TILE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t oq = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
          umma_ss_lh(d, qa + oq, s_hi, kb + oq, s_hi, C::IDESC_S, kk ? 1u : 0u);
        }
        umma_commit(&s_full[g & 1]);
        umma_commit(&kv_empty[kslot]);                  // K read
        if (n == NB - 1) umma_commit(&q_empty[qs]);     // the tile's Q read by its last S
        return true;
      };
      // O_seg (+)= P V of block g; the tile's first P V waits until the epilogue has read O
      auto issue_pv = [&](int g) -> bool {
        const int li = g / NB, n = g % NB;
        const int sg = n < nb0 ? 0 : 1;
        const bool first = (n == 0) || (n == nb0);
        if (n == 0 && li > 0) {
          if (!mbar_wait(o_free, (li - 1) & 1u, SITE_OF)) return false;
          tc_fence_after();
        }
        const int vseq = 2 * g + 1, vslot = vseq % RING;
        const uint32_t d = tmem + o_col(sg), pa = tmem + s_col(g);
        const uint32_t vb = v_lo + vslot * (TILE_BYTES >> 4);
#pragma unroll
        for (int part = 0; part < PP; ++part) {
          if (!mbar_wait(part == 0 ? &p_part[g & 1] : &p_full[g & 1], (g >> 1) & 1u, SITE_P)) return false;
          if (part == 0 && !mbar_wait(&kv_full[vslot], (vseq / RING) & 1u, SITE_KVF)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = part * 4; kk < part * 4 + 4; ++kk)   // 16 keys = 8 TMEM columns of P; 2048 bytes of V
            umma_ts_lh(d, pa + 8 * kk, vb + kk * (2048 >> 4), v_hi, C::IDESC_O, (!first || kk) ? 1u : 0u);
        }
        umma_commit(&pv_done[g & 1]);
        umma_commit(&kv_empty[vslot]);                  // V read
        if (n == NB - 1) umma_commit(o_done);           // the tile's O complete
        return true;
      };
      // S of two blocks ahead; then per block its P V and S of the block two ahead
      // (the MMAs of this thread run in issue order, so S never overwrites a P
      // that an issued P V still has to read)
      for (int g = 0; g < 2 && g < G && ok; ++g) ok = issue_s(g);
      for (int g = 0; g < G && ok; ++g) {
        ok = issue_pv(g);
        if (ok && g + 2 < G) ok = issue_s(g + 2);
      }
      umma_commit(tdone);
      mbar_wait(tdone, 0, SITE_DRAIN);
    }
    __syncwarp();
  }
  else if (warp < 6) {
    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;     // query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    int g = 0;
    for (int li = 0; li < n_items && ok; ++li) {
      float m = -INFINITY, l = 0.f, l_first = 0.f;
      for (int n = 0; n < NB; ++n, ++g) {
        const int sg = n < nb0 ? 0 : 1;
        const bool first = (n == 0) || (n == nb0);
        if (n == nb0) { l_first = l; m = -INFINITY; l = 0.f; }
        const uint32_t s_addr = tmem + lane_base + s_col(g);
        if (!mbar_wait_warp(&s_full[g & 1], (g >> 1) & 1u, SITE_S)) { ok = false; break; }
        tc_fence_after();
        const int valid = (sg ? nk1 : nk0) - (n - (sg ? nb0 : 0)) * BK;   // keys of this block that exist
        uint32_t a[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, a[c]);
        tmem_wait_ld();
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
        const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * p.scale_log2;
        // lazy rescale: the reference moves only when the block's maximum exceeds it by the threshold
        const bool grow = mx > m + RESCALE_THRESHOLD;
        const float m_new = grow ? mx : m;
        const float alpha = grow ? tca::ex2(m - m_new) : 1.f;
        m = m_new;
        if (__any_sync(0xffffffffu, grow) && !first) {
          // O_seg *= alpha once P V of the previous block (issued after this block's S) has completed
          if (!mbar_wait_warp(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1u, SITE_O)) { ok = false; break; }
          tc_fence_after();
          const uint32_t o_addr = tmem + lane_base + o_col(sg);
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
        // P = 2^(s scale - m) in the operand type over the block's S columns (chunk c of 16 keys
        // -> 8 columns at 8c), released to P V in two halves
        float2 rs4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(-m, -m);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const int kk = (c & 1) * 16 + k;
            const float2 arg = ffma2(make_float2(__uint_as_float(a[c >> 1][kk]), __uint_as_float(a[c >> 1][kk + 1])),
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
          tmem_st8(s_addr + c * 8, pk);
          if (c == 3) {   // keys 0..63 written
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_part[g & 1]);
          }
        }
        tmem_wait_st();
        const float2 rs = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
        l = l * alpha + (rs.x + rs.y);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g & 1]);
      }
      if (!ok) break;
      // the tile's row sums for the epilogue warps (the next tile's sums are written only
      // after its P V has waited for this tile's epilogue to read O)
      st[r] = l;
      st[128 + r] = l_first;
      __syncwarp();
      if (lane == 0) mbar_arrive(st_full);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // out = O_text / l + O_image / l_first, rounded to bf16
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    for (int li = 0; li < n_items; ++li) {
      int qb, h, b;
      tile_of(li, qb, h, b);
      if (!mbar_wait_warp(st_full, li & 1u, SITE_ST)) break;
      if (!mbar_wait_warp(o_done, li & 1u, SITE_O)) break;
      tc_fence_after();
      const float inv1 = 1.f / st[r], inv0 = 1.f / st[128 + r];
      const int row = qb * BQ + r;
      bf16* dst = p.o + (static_cast<int64_t>(b) * p.Lq + row) * p.o_rs + h * DH;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        float v[32];
        tmem_ld32(tmem + lane_base + o_col(1) + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(o[k]) * inv1;
        tmem_ld32(tmem + lane_base + o_col(0) + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] += __uint_as_float(o[k]) * inv0;
        if (row < p.Lq) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                               pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace tcx

// ------------------------------------------------------------------ host side
// Two key segments (k1/v1 and k2/v2), head dim 128, one CTA per SM (or per tile
// when there are fewer tiles), each looping over Q tiles of 128 rows.
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
  p.heads = a.heads;
  p.batch = a.batch;
  p.nqb = (a.Lq + tcx::BQ - 1) / tcx::BQ;
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
  const int64_t items = static_cast<int64_t>(p.nqb) * a.heads * a.batch;
  if (items > 0x7fffffff) { set_error("cross-attention: too many tiles"); return WD_ERR_SHAPE; }
  const int grid = items < sm_count() ? static_cast<int>(items) : sm_count();
  Trace tr(a.cross ? KC_ATTN_CROSS : KC_ATTN_SELF, st);
  tcx::k_attn_cross<TI><<<grid, tcx::THREADS, tcx::SMEM, st>>>(tq, tk0, tv0, tk1, tv1, p);
  return launch_status("attention_cross_tc");
}
template wd_status attention_cross_tc<bf16>(const AttnArgs<bf16, bf16>&, cudaStream_t);
template wd_status attention_cross_tc<f16>(const AttnArgs<f16, bf16>&, cudaStream_t);

}  // namespace wd
