// k_attn_tc.cu — non-causal multi-head attention on the sm_100a tensor cores
// (tcgen05 + TMEM + TMA), head dim 128, bf16 or IEEE half operands (q, k, v
// and the probabilities P share one type), bf16 out, fp32 softmax and
// accumulation ("图解 Wan2.1 I2V" 5.3: full spatio-temporal self-attention;
// 5.4: decoupled image/text cross-attention, two softmaxes summed).
//
// A CTA owns NQ query tiles of 128 rows of one (batch, head) and streams the
// keys/values of NSEG segments in 128-key blocks:
//   warp 0           TMA loader: the Q tiles once, then K_j, V_j through a
//                    ring of RING 32 KB tiles
//   warp 1           TMEM owner + MMA issuer: S_t = Q_t K_j^T into TMEM,
//                    O_t (+)= P_t V_j with P_t read from TMEM (TS form), so
//                    this product reads only V from shared memory; P V is
//                    issued in two 64-key halves as the softmax writes P
//   warps 2..        4 * SPLIT softmax warps per Q tile, SPLIT per TMEM lane
//                    quarter (32 query rows), each owning 128 / SPLIT key
//                    columns (SPLIT = 1 by default: one thread holds a whole
//                    row of S in registers, so no row maxima are exchanged).
//                    Online softmax on S_t read from TMEM, P_t written back
//                    over the warp's own S columns, O_t rescaled in TMEM
//                    only when the running max grows by more than 8 (log2
//                    units; the final 1/l keeps the result exact), then the
//                    normalised output written out.
// With NQ = 2 the two tiles ping-pong: while one tile's warps run their
// softmax, the tensor cores compute the other tile's P V and next S.  With
// two key segments (one Q tile: its O and O' take half of TMEM) S is double
// buffered instead: S of block n + 1 is computed while the softmax works on
// block n, and P V of block n runs while it works on block n + 1.
#include "wd_internal.cuh"

namespace wd {
namespace tca {

constexpr int BQ = 128, DH = 128;
constexpr int TILE_BYTES = 128 * 128 * 2;   // one 128 x 128 Q tile of 2-byte elements (two 64-column halves)
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int RING_BYTES = 4 * TILE_BYTES;  // K/V tiles in flight: 128 KB of shared memory
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units

#ifndef WD_ATTN_SELF_BK
#define WD_ATTN_SELF_BK 128   // keys per block of the self-attention (128, or 64 with double-buffered S)
#endif

#ifndef WD_ATTN_P_PARTS
#define WD_ATTN_P_PARTS 2   // releases of a block's P to its P V (one softmax warp per lane quarter): 1, 2 or 4
#endif

#ifndef WD_ATTN_ILP
#define WD_ATTN_ILP 1   // 1: row max and row sum over four independent chains (shorter dependency chains)
#endif

#ifndef WD_ATTN_SPEC
#define WD_ATTN_SPEC 0   // 1: no separate row-max pass before the exponentials (speculative reference)
#endif

#ifndef WD_ATTN_ISSUERS
#define WD_ATTN_ISSUERS 1   // MMA issuing threads of the self-attention (1, or 2: one per Q tile)
#endif

#ifndef WD_ATTN_SPLIT
#define WD_ATTN_SPLIT 1   // softmax warps per TMEM lane quarter (1 or 2), each owning 128/SPLIT key columns
#endif
constexpr int SPLIT = WD_ATTN_SPLIT;
static_assert(SPLIT == 1 || SPLIT == 2, "WD_ATTN_SPLIT must be 1 or 2");

template <int NQ, int NSEG, typename TI, int BK = 128>
struct Cfg {
  static_assert(BK == 128 || BK == 64, "keys per block: 128 or 64");
  static constexpr int BKV = BK;
  // one K or V tile: BK keys x 128 dims, stored as two 64-dim halves of BK rows x 128 bytes
  static constexpr int KV_BYTES = BK * DH * 2;
  static constexpr int KV_HALF = KV_BYTES / 2;
  static constexpr int RING = RING_BYTES / KV_BYTES;
  // 2 warps (loader, MMA) + per Q tile 4*SPLIT softmax warps: SPLIT per TMEM
  // lane quarter (32 query rows), each owning BK/SPLIT of the key columns.
  static constexpr int SM_WARPS = 4 * SPLIT;
  static constexpr int COLS = BKV / SPLIT;
  static_assert(COLS % 64 == 0, "each softmax warp owns a multiple of 64 key columns");
  // P of a block is handed to its P V in PP parts (each part's k-steps start once it is in TMEM)
  static constexpr int PP = SPLIT == 1 ? WD_ATTN_P_PARTS : 1;
  static_assert(PP == 1 || PP == 2 || PP == 4, "P released in 1, 2 or 4 parts");
  static constexpr int PPB = PP > 1 ? PP - 1 : 1;   // barriers for the parts before the last
  // speculative softmax (see the softmax warps): one thread per row, P released in at most two parts
  static constexpr bool SPEC = WD_ATTN_SPEC && SPLIT == 1 && PP <= 2 && WD_ATTN_ILP;
  // MMA issuing threads: one for all tiles, or (two tiles of one segment) one per tile,
  // so that one issuer's waits overlap the other's MMAs
  static constexpr int ISSUERS = (NSEG == 1 && NQ == 2) ? WD_ATTN_ISSUERS : 1;
  static_assert(ISSUERS == 1 || ISSUERS == NQ, "one issuer, or one per Q tile");
  static constexpr int THREADS = 32 * (1 + ISSUERS) + 32 * SM_WARPS * NQ;
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NQ * TILE_BYTES;
  static constexpr int XCH_OFF = RING_OFF + RING_BYTES;     // row-max / row-sum exchange
  static constexpr int XCH_BYTES = NQ * (2 * 2 * 128 + 2 * 2 * 128) * 4;
  static constexpr int BAR_OFF = XCH_OFF + XCH_BYTES;
  static constexpr int SMEM = 1024 + BAR_OFF + 512;
  static_assert(SMEM <= 232448, "shared memory budget of one CTA exceeded");
  static constexpr int TMEM_COLS = 512;
  // TMEM columns (512):
  //  - one segment, 128-key blocks: S_t, O_t per tile (two tiles), one S buffer each;
  //  - one segment, 64-key blocks: O_0, O_1 in columns 0-255, then two 64-column S
  //    buffers per tile, so that S of block n + 1 is computed while the softmax
  //    works on block n (double buffering);
  //  - two segments (one tile): O and O' in the middle and two 128-column S buffers.
  static constexpr bool DB = NSEG == 2 || BK == 64;   // double-buffered S
  static_assert(NSEG == 1 || (NQ == 1 && BK == 128), "two key segments use one Q tile of 128-key blocks");
  static constexpr int NBUF = DB ? 2 * NQ : NQ;   // S/P buffers (and their barriers)
  __host__ __device__ static constexpr int buf(int t, int n) { return DB ? 2 * t + (n & 1) : t; }
  __host__ __device__ static constexpr uint32_t par(int n) { return DB ? ((n >> 1) & 1u) : (n & 1u); }
  __host__ __device__ static constexpr int s_col(int t, int n) {
    return NSEG == 2 ? ((n & 1) ? 384 : 0) : (BK == 64 ? 256 + 128 * t + 64 * (n & 1) : t * 256);
  }
  __host__ __device__ static constexpr int o_col(int t, int seg) {
    return NSEG == 2 ? 128 + 128 * seg : (BK == 64 ? 128 * t : t * 256 + 128);
  }
  // Q K^T: both K-major; P V: P from TMEM, V MN-major (dh contiguous).  P is
  // held in the operands' type (A and B of one MMA share their type).
  static constexpr bool HALF = std::is_same<TI, f16>::value;
  static constexpr uint32_t IDESC_S = HALF ? idesc_f16(128, BK, 0, 0) : idesc_bf16(128, BK, 0, 0);
  static constexpr uint32_t IDESC_O = HALF ? idesc_f16(128, 128, 0, 1) : idesc_bf16(128, 128, 0, 1);
};

enum : unsigned { SITE_Q = 0x201, SITE_KVF = 0x202, SITE_KVE = 0x203, SITE_S = 0x204, SITE_P = 0x205,
                  SITE_O = 0x206, SITE_DRAIN = 0x207 };

struct Seg {
  int n;        // keys
  int shared;   // keys shared by the batch (tensor map batch extent 1)
};

// Every tensor map starts at its operand's first column, so head h's columns
// are [h*128, h*128 + 128) in all of them.
struct Params {
  int Lq;       // query rows per batch
  Seg seg[2];
  bf16* o;
  int64_t o_rs;
  float scale_log2;
  float* lse;   // one segment, optional: [batch, heads, Lq] row log-sum-exp (log2 units)
  int heads;
};

// Bounded waits: the MMA thread alone, the softmax warps as whole warps.
#define MMA_WAIT(bar, par, site) mbar_wait(bar, par, site)
#define SM_WAIT(bar, par, site) mbar_wait_warp(bar, par, site)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA/ALU pipes, to take part of the exponentials off the MUFU
// unit (the softmax otherwise saturates it at the same rate as the tensor
// cores).  Range reduction x = j + f with j = round(x): adding 1.5 * 2^23
// leaves round(x) in the low mantissa bits of the sum (round-to-nearest-even);
// 2^f on [-1/2, 1/2] is a degree-3 polynomial whose coefficients were fitted
// for this library (iteratively reweighted least squares on the relative
// error, max relative error 7.5e-5 in fp32, far below a bf16 half-ulp); the
// factor 2^j is added to the exponent field.  Arguments below -125 give 2^-125 (~0).
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.f);   // keeps q * 2^round(x) a normal float (q >= 0.7)
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  const float q = fmaf(fmaf(fmaf(0.0551716648f, f, 0.2426111251f), f, 0.6932609677f), f, 0.9999280572f);
  // round(x) sits in the low bits of t's encoding; 0x4B400000 << 23 is 0 mod 2^32
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

// The same on two lanes at once with the packed fp32 instructions (f32x2): each
// lane's operations and roundings are those of exp2_fma, in fewer instructions.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 magic = make_float2(12582912.f, 12582912.f);
  const float2 t = fadd2(x, magic);
  const float2 f = fsub2(x, fsub2(t, magic));
  const float2 c3 = make_float2(0.0551716648f, 0.0551716648f), c2 = make_float2(0.2426111251f, 0.2426111251f);
  const float2 c1 = make_float2(0.6932609677f, 0.6932609677f), c0 = make_float2(0.9999280572f, 0.9999280572f);
  const float2 q = ffma2(ffma2(ffma2(c3, f, c2), f, c1), f, c0);
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

#ifndef WD_EXP2_PACKED
#define WD_EXP2_PACKED 1   // 1: the FMA-pipe exponentials of a pair of keys in one packed evaluation
#endif

#ifndef WD_EXP2_EMU_PER8
#define WD_EXP2_EMU_PER8 2   // of every 8 exponentials, this many run on the FMA pipe
#endif

template <int NQ, int NSEG, typename TI, int BK>
__global__ void __launch_bounds__(Cfg<NQ, NSEG, TI, BK>::THREADS, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK0,
          const __grid_constant__ CUtensorMap tmV0, const __grid_constant__ CUtensorMap tmK1,
          const __grid_constant__ CUtensorMap tmV1, const Params p) {
  using C = Cfg<NQ, NSEG, TI, BK>;
  constexpr int RING = C::RING, BKV = C::BKV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;                 // 1
  uint64_t* kv_full = bars + 1;            // RING
  uint64_t* kv_empty = kv_full + RING;     // RING
  uint64_t* s_full = kv_empty + RING;      // NBUF
  uint64_t* p_full = s_full + C::NBUF;     // NBUF: all of P written
  uint64_t* p_part = p_full + C::NBUF;     // NBUF x PPB: the first parts of the block's P written
  uint64_t* pv_done = p_part + C::NBUF * C::PPB;   // NBUF: P V of the block in that buffer completed (double buffering)
  uint64_t* o_done = pv_done + C::NBUF;    // NQ
  uint64_t* tdone = o_done + NQ;           // 1
  uint64_t* mx_bar = tdone + 1;            // NQ x 4: the two warps of a lane quarter swap row maxima
  uint64_t* fin_bar = mx_bar + 4 * NQ;     // NQ x 4: ... and their row sums at the end
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin_bar + 4 * NQ);
  float* xmax = reinterpret_cast<float*>(smem + C::XCH_OFF);   // [2 parity][NQ][2 halves][128 rows]
  float* xsum = xmax + 2 * NQ * 2 * 128;                        // [NQ][2 halves][2 (l, l_first)][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int l0 = qb * BQ * NQ;
  const int nk0 = p.seg[0].n, nk1 = p.seg[1].n;
  const int sh0 = p.seg[0].shared, sh1 = p.seg[1].shared;
  const int nb0 = (nk0 + BKV - 1) / BKV;
  const int nb1 = NSEG == 2 ? (nk1 + BKV - 1) / BKV : 0;
  const int NB = nb0 + nb1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < RING; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], C::ISSUERS); }
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::SM_WARPS);
      for (int j = 0; j < C::PPB; ++j) mbar_init(&p_part[i * C::PPB + j], C::SM_WARPS);
      mbar_init(&pv_done[i], 1);
    }
    for (int t = 0; t < NQ; ++t) mbar_init(&o_done[t], 1);
    mbar_init(tdone, C::ISSUERS);
    for (int i = 0; i < 4 * NQ; ++i) { mbar_init(&mx_bar[i], 2); mbar_init(&fin_bar[i], 2); }
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loader
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0, last_par = 0;
      mbar_arrive_expect_tx(q_full, NQ * TILE_BYTES);
      for (int t = 0; t < NQ; ++t)
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + C::Q_OFF + t * TILE_BYTES + hf * HALF_BYTES, &tmQ, h * DH + hf * 64,
                      l0 + t * BQ, b, q_full);
      for (int n = 0; n < NB && ok; ++n) {
        const int sg = n < nb0 ? 0 : 1;
        const int j0 = (n - (sg ? nb0 : 0)) * BKV;
        const CUtensorMap* tk = sg ? &tmK1 : &tmK0;
        const CUtensorMap* tv = sg ? &tmV1 : &tmV0;
        const int bb = (sg ? sh1 : sh0) ? 0 : b;
        for (int kv = 0; kv < 2; ++kv) {
          const int seq = 2 * n + kv, slot = seq % RING;
          const uint32_t ph = (seq / RING) & 1u;
          if (!mbar_wait(&kv_empty[slot], ph ^ 1u, SITE_KVE)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[slot], C::KV_BYTES);
          const int col = h * DH;
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(smem + C::RING_OFF + slot * C::KV_BYTES + hf * C::KV_HALF, kv ? tv : tk, col + hf * 64, j0,
                        bb, &kv_full[slot]);
          issued |= 1u << slot;
          last_par = (last_par & ~(1u << slot)) | (ph << slot);
        }
      }
      mbar_wait(q_full, 0, SITE_DRAIN);
      for (int s = 0; s < RING; ++s)
        if (issued & (1u << s)) mbar_wait(&kv_full[s], (last_par >> s) & 1u, SITE_DRAIN);
    }
    __syncwarp();
  } else if (warp <= C::ISSUERS) {
    // ------------------------------------------------------------ MMA issuer(s)
    // tiles [t_lo, t_hi) of this issuer: all of them, or its own one
    const int t_lo = C::ISSUERS == 1 ? 0 : warp - 1, t_hi = C::ISSUERS == 1 ? NQ : warp;
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, SITE_Q);
      tc_fence_after();
      const uint32_t q0 = smem_u32(smem + C::Q_OFF);
      const uint32_t r0 = smem_u32(smem + C::RING_OFF);
      // Shared-memory descriptors as (low, high) halves: the high halves are
      // fixed, the start address in the low half steps by 16-byte units.
      const uint64_t dq0 = sdesc_sw128(q0, 16, 1024), dk0 = sdesc_sw128(r0, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(r0, C::KV_HALF, 1024);
      const uint32_t q_lo = static_cast<uint32_t>(dq0), k_lo = static_cast<uint32_t>(dk0);
      const uint32_t v_lo = static_cast<uint32_t>(dv0);
      const uint32_t s_hi = static_cast<uint32_t>(dq0 >> 32), v_hi = static_cast<uint32_t>(dv0 >> 32);
      // P_t V_j for block n of tile t
      auto issue_pv = [&](int t, int n) -> bool {
        const int vseq = 2 * n + 1, vslot = vseq % RING;
        const int sg = n < nb0 ? 0 : 1;
        const int first = (n == 0) || (n == nb0);
        const int bi = C::buf(t, n);
        const uint32_t d = tmem + C::o_col(t, sg);
        const uint32_t pa = tmem + C::s_col(t, n), vb_lo = v_lo + vslot * (C::KV_BYTES >> 4);
        // P arrives in PP parts of the block's keys: the k-steps of a part start as
        // soon as that part is in TMEM.
        constexpr int KK = BKV / 16;
#pragma unroll
        for (int part = 0; part < C::PP; ++part) {
          uint64_t* bar = part < C::PP - 1 ? &p_part[bi * C::PPB + part] : &p_full[bi];
          if (!MMA_WAIT(bar, C::par(n), SITE_P)) return false;
          // the V tile: waited for by this issuer's first tile (its other tiles read the same tile)
          if (part == 0 && t == t_lo && !MMA_WAIT(&kv_full[vslot], (vseq / RING) & 1u, SITE_KVF)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = part * KK / C::PP; kk < (part + 1) * KK / C::PP; ++kk) {
            // A = P: 16 keys = 8 TMEM columns of packed bf16 pairs; each softmax
            // warp's keys sit over the first half of its own S columns:
            // key 16 kk lives at column (16kk / COLS) * COLS + (16kk % COLS) / 2
            // B = V rows 16 kk .. 16 kk + 15: 2048 bytes on within each 64-dim half
            umma_ts_lh(d, pa + (16 * kk / C::COLS) * C::COLS + (16 * kk % C::COLS) / 2, vb_lo + kk * (2048 >> 4), v_hi,
                       C::IDESC_O, (!first || kk) ? 1u : 0u);
          }
        }
        if (C::DB) umma_commit(&pv_done[bi]);
        if (t == t_hi - 1) umma_commit(&kv_empty[vslot]);
        return true;
      };
      // S_t = Q_t K_n^T into tile t's S buffer for block n (K tile already waited for)
      auto issue_s = [&](int t, int n) {
        const int kslot = (2 * n) % RING;
        const uint32_t d = tmem + C::s_col(t, n);
        const uint32_t qa = q_lo + t * (TILE_BYTES >> 4), kb = k_lo + kslot * (C::KV_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          // 16 dims per step: 32 bytes into a 128-byte row of the step's 64-dim half
          const uint32_t oq = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
          const uint32_t ok_ = ((kk >> 2) * C::KV_HALF + (kk & 3) * 32) >> 4;
          umma_ss_lh(d, qa + oq, s_hi, kb + ok_, s_hi, C::IDESC_S, kk ? 1u : 0u);
        }
        umma_commit(&s_full[C::buf(t, n)]);
      };
      auto wait_k = [&](int n) -> bool {
        const int kseq = 2 * n;
        if (!MMA_WAIT(&kv_full[kseq % RING], (kseq / RING) & 1u, SITE_KVF)) return false;
        tc_fence_after();
        return true;
      };
      if constexpr (C::DB) {
        // Two S buffers per tile: S of blocks 0 and 1 first; then per block and
        // tile P V, and S of the block two ahead into the buffer that P V has
        // read (the MMAs of one thread run in issue order).
        for (int n = 0; n < 2 && n < NB && ok; ++n) {
          if (!wait_k(n)) { ok = false; break; }
          for (int t = t_lo; t < t_hi; ++t) issue_s(t, n);
          umma_commit(&kv_empty[(2 * n) % RING]);
        }
        for (int n = 0; n < NB && ok; ++n) {
          for (int t = t_lo; t < t_hi && ok; ++t) {
            if (!issue_pv(t, n)) { ok = false; break; }
            if (n + 2 < NB) {
              if (t == t_lo && !wait_k(n + 2)) { ok = false; break; }
              issue_s(t, n + 2);
            }
          }
          if (ok && n + 2 < NB) umma_commit(&kv_empty[(2 * (n + 2)) % RING]);
        }
        for (int t = t_lo; t < t_hi && ok; ++t) umma_commit(&o_done[t]);
      } else {
        for (int n = 0; n < NB && ok; ++n) {
          for (int t = t_lo; t < t_hi && ok; ++t) {
            // P_t V of the previous block first: it needs only P_t and that V tile,
            // not the next K tile.
            if (n > 0 && !issue_pv(t, n - 1)) { ok = false; break; }
            if (t == t_lo && !wait_k(n)) { ok = false; break; }
            issue_s(t, n);
          }
          if (ok) umma_commit(&kv_empty[(2 * n) % RING]);
        }
        for (int t = t_lo; t < t_hi && ok; ++t) {
          if (!issue_pv(t, NB - 1)) { ok = false; break; }
          umma_commit(&o_done[t]);
        }
      }
      umma_commit(tdone);
      mbar_wait(tdone, 0, SITE_DRAIN);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    constexpr int COLS = C::COLS, CH = COLS / 32;      // this warp's key columns of a block
    constexpr int OCOLS = DH / SPLIT, OCH = OCOLS / 32;   // ... and its output columns (of dh)
    const int sw = warp - 1 - C::ISSUERS;
    const int t = sw / C::SM_WARPS;        // Q tile
    const int hc = SPLIT == 2 ? (sw >> 2) & 1 : 0;   // key part of this warp: columns [COLS hc, COLS hc + COLS)
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;     // query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    [[maybe_unused]] uint64_t* my_mx = &mx_bar[t * 4 + quarter];
    float m = -INFINITY, l = 0.f, l_first = 0.f;
    bool ok = true;
    for (int n = 0; n < NB; ++n) {
      const int sg = n < nb0 ? 0 : 1;
      const bool first = (n == 0) || (n == nb0);
      if (NSEG == 2 && n == nb0) { l_first = l; m = -INFINITY; l = 0.f; }
      const int bi = C::buf(t, n);
      const uint32_t s_addr = tmem + lane_base + C::s_col(t, n) + hc * COLS;
      if (!SM_WAIT(&s_full[bi], C::par(n), SITE_S)) { ok = false; break; }
      tc_fence_after();
      // keys of this block that exist, counted from this warp's first column
      const int valid = (sg ? nk1 : nk0) - (n - (sg ? nb0 : 0)) * BKV - hc * COLS;
      const bool ragged = valid < COLS;                                     // warp-uniform
      // one read of this warp's score columns; they stay in registers
      uint32_t a[CH][32];
#pragma unroll
      for (int c = 0; c < CH; ++c) tmem_ld32(s_addr + c * 32, a[c]);
      tmem_wait_ld();
      if (ragged) {
#pragma unroll
        for (int c = 0; c < CH; ++c)
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (c * 32 + k >= valid) a[c][k] = __float_as_uint(-INFINITY);
      }
      // exponentials of 16-key chunk c against the reference -nm2, packed into TMEM over this
      // warp's own S columns (chunk c -> 8 columns at 8c), summed into rs4 / rs2
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      auto emit = [&](int c, float2 nm2, float2 (&rs4)[4], float2& rs2) {
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const int kk = (c & 1) * 16 + k;
          const float2 arg = ffma2(make_float2(__uint_as_float(a[c >> 1][kk]), __uint_as_float(a[c >> 1][kk + 1])),
                                   sc2, nm2);
          float e0, e1;
          if (WD_EXP2_PACKED && (k & 7) >= 8 - WD_EXP2_EMU_PER8 && ((k + 1) & 7) >= 8 - WD_EXP2_EMU_PER8) {
            const float2 e = exp2_fma2(arg);
            e0 = e.x;
            e1 = e.y;
          } else {
            e0 = ((k & 7) >= 8 - WD_EXP2_EMU_PER8) ? exp2_fma(arg.x) : ex2(arg.x);
            e1 = (((k + 1) & 7) >= 8 - WD_EXP2_EMU_PER8) ? exp2_fma(arg.y) : ex2(arg.y);
          }
          if constexpr (WD_ATTN_ILP) rs4[(k >> 1) & 3] = fadd2(rs4[(k >> 1) & 3], make_float2(e0, e1));
          else rs2 = fadd2(rs2, make_float2(e0, e1));
          pk[k >> 1] = C::HALF ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
        }
        tmem_st8(s_addr + c * 8, pk);
      };
      // O_t *= alpha on this warp's output columns for rows whose reference max moved,
      // before any of this block's P V can start.  With one S buffer per tile, P V of
      // the previous block has completed (its commit precedes the S commit waited on);
      // with two, S of this block was issued before that P V, so wait for it.
      auto rescale_o = [&](float alpha) -> bool {
        if (C::DB && !mbar_wait_warp(&pv_done[C::buf(t, n - 1)], C::par(n - 1), SITE_O)) return false;
        if (C::DB) tc_fence_after();
        const uint32_t o_addr = tmem + lane_base + C::o_col(t, sg) + hc * OCOLS;
#pragma unroll 1
        for (int c = 0; c < OCH; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(o_addr + c * 32, o);
        }
        tmem_wait_st();
        return true;
      };
      if constexpr (C::SPEC) {
        if (!first) {
          // Speculative pass: the first half's exponentials run against the current
          // reference m while the row maximum is taken beside them (no pass before).
          // The maximum is checked before that half's P is released; if a row's grew
          // past the threshold, the warp moves those rows' reference, rescales O and
          // redoes the half, so P, l and O end as with the maximum taken first.
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < CH; c += 2)
#pragma unroll
            for (int k = 0; k < 32; k += 2)
              m4[(k >> 1) & 3] = fmax3(m4[(k >> 1) & 3],
                                       fmax3(__uint_as_float(a[c][k]), __uint_as_float(a[c][k + 1]),
                                             __uint_as_float(a[c + 1][k])),
                                       __uint_as_float(a[c + 1][k + 1]));
          float2 rs2s = make_float2(0.f, 0.f);
          float2 rs4s[4] = {rs2s, rs2s, rs2s, rs2s};
          float2 nm2 = make_float2(-m, -m);
#pragma unroll
          for (int c = 0; c < CH; ++c) emit(c, nm2, rs4s, rs2s);
          const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * p.scale_log2;
          const bool grow = mx > m + RESCALE_THRESHOLD;
          float alpha = 1.f;
          if (__any_sync(0xffffffffu, grow)) {
            const float m_new = grow ? mx : m;
            alpha = grow ? ex2(m - m_new) : 1.f;
            m = m_new;
            tmem_wait_st();   // the first half's stores land before they are rewritten
            if (!rescale_o(alpha)) { ok = false; break; }
            nm2 = make_float2(-m, -m);
#pragma unroll
            for (int j = 0; j < 4; ++j) rs4s[j] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < CH; ++c) emit(c, nm2, rs4s, rs2s);
          }
          if constexpr (C::PP == 2) {   // the first half of P is written: release its P V
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_part[bi * C::PPB]);
          }
#pragma unroll
          for (int c = CH; c < 2 * CH; ++c) emit(c, nm2, rs4s, rs2s);
          tmem_wait_st();
          const float2 rsum = fadd2(fadd2(rs4s[0], rs4s[1]), fadd2(rs4s[2], rs4s[3]));
          l = l * alpha + (rsum.x + rsum.y);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[bi]);
          continue;
        }
      }
      float mx = -INFINITY;
      if constexpr (WD_ATTN_ILP) {
        // four chains, each over every fourth pair of columns, then combined
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < CH; c += 2)
#pragma unroll
          for (int k = 0; k < 32; k += 2)
            m4[(k >> 1) & 3] = fmax3(m4[(k >> 1) & 3],
                                     fmax3(__uint_as_float(a[c][k]), __uint_as_float(a[c][k + 1]),
                                           __uint_as_float(a[c + 1][k])),
                                     __uint_as_float(a[c + 1][k + 1]));
        mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
      } else {
#pragma unroll
        for (int c = 0; c < CH; c += 2)
#pragma unroll
          for (int k = 0; k < 32; k += 2)
            mx = fmax3(mx, fmax3(__uint_as_float(a[c][k]), __uint_as_float(a[c][k + 1]), __uint_as_float(a[c + 1][k])),
                       __uint_as_float(a[c + 1][k + 1]));
      }
      if constexpr (SPLIT == 2) {   // the two warps of a lane quarter swap their row maxima
        float* slot = xmax + ((n & 1) * NQ + t) * 256;
        slot[hc * 128 + r] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(my_mx);
        if (!SM_WAIT(my_mx, n & 1u, SITE_S)) { ok = false; break; }
        mx = fmaxf(mx, slot[(1 - hc) * 128 + r]);
      }
      mx *= p.scale_log2;
      // lazy rescale: move the reference max only when it grew by more than the threshold
      const bool grow = mx > m + RESCALE_THRESHOLD;
      const float m_new = grow ? mx : m;
      const float alpha = grow ? ex2(m - m_new) : 1.f;
      m = m_new;
      const float neg_m = -m;
      if (__any_sync(0xffffffffu, grow) && !first && !rescale_o(alpha)) { ok = false; break; }
      // P = exp2(s * scale - m) as packed pairs (operand type) into TMEM over this warp's
      // own S columns: chunk c of 16 keys -> 8 columns at 8c (masked keys hold
      // -inf, so their exponential is 0)
      float2 rs2 = make_float2(0.f, 0.f);
      [[maybe_unused]] float2 rs4[4] = {rs2, rs2, rs2, rs2};   // four partial sums (WD_ATTN_ILP)
      const float2 nm2 = make_float2(neg_m, neg_m);
#pragma unroll
      for (int c = 0; c < 2 * CH; ++c) {
        emit(c, nm2, rs4, rs2);
        if constexpr (C::PP > 1) {   // a part of the block's P is written: release its P V
          constexpr int per = 2 * CH / C::PP;   // 16-key chunks per part
          if ((c + 1) % per == 0 && c + 1 < 2 * CH) {
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_part[bi * C::PPB + (c + 1) / per - 1]);
          }
        }
      }
      tmem_wait_st();
      if constexpr (WD_ATTN_ILP) rs2 = fadd2(fadd2(rs4[0], rs4[1]), fadd2(rs4[2], rs4[3]));
      l = l * alpha + (rs2.x + rs2.y);     // this warp's share of the row sum
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[bi]);
    }
    // ---------------------------------------------------------- epilogue
    if (SPLIT == 2 && ok) {
      // combine the two parts' row sums
      float* xs = xsum + t * 512;
      xs[hc * 256 + r] = l;
      xs[hc * 256 + 128 + r] = l_first;
      __syncwarp();
      if (lane == 0) mbar_arrive(&fin_bar[t * 4 + quarter]);
      ok = mbar_wait_warp(&fin_bar[t * 4 + quarter], 0, SITE_O);
      if (ok) {
        l += xs[(1 - hc) * 256 + r];
        l_first += xs[(1 - hc) * 256 + 128 + r];
      }
    }
    if (ok && mbar_wait_warp(&o_done[t], 0, SITE_O)) {
      tc_fence_after();
      const int row = l0 + t * BQ + r;
      const float inv1 = 1.f / l;
      // the row's log-sum-exp in log2 units: the reference max plus log2 of the sum relative to it
      if (NSEG == 1 && p.lse && hc == 0 && row < p.Lq)
        p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.Lq + row] = m + __log2f(l);
      const float inv0 = NSEG == 2 ? 1.f / l_first : 0.f;
      bf16* dst = p.o + (static_cast<int64_t>(b) * p.Lq + row) * p.o_rs + h * DH + hc * OCOLS;
#pragma unroll 1
      for (int c = 0; c < OCH; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + C::o_col(t, NSEG - 1) + hc * OCOLS + c * 32, o);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(o[k]) * inv1;
        if (NSEG == 2) {
          uint32_t o2[32];
          tmem_ld32(tmem + lane_base + C::o_col(t, 0) + hc * OCOLS + c * 32, o2);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] += __uint_as_float(o2[k]) * inv0;
        }
        if (row < p.Lq) {
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
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace tca

// ------------------------------------------------------------------ host side
// 3D tensor map (bf16 or IEEE half elements) over [batches, rows, cols] (cols contiguous, row stride
// `rs` elements, batch stride `bs` elements); box = 64 cols x box_rows rows x 1.
static wd_status make_tmap_3d(CUtensorMap* m, CUtensorMapDataType type, const void* base, int64_t cols, int64_t rows,
                              int64_t batches, int64_t rs, int64_t bs, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) { set_error("cuTensorMapEncodeTiled unavailable"); return WD_ERR_CUDA; }
  if (batches > 1 && (bs * 2) % 16) { set_error("attention: batch stride not 16-byte aligned"); return WD_ERR_ALIGN; }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batches)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(rs) * 2,
                           static_cast<cuuint64_t>(batches > 1 ? bs : rs * rows) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, type, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { set_error("cuTensorMapEncodeTiled (3d) failed (%d)", static_cast<int>(r)); return WD_ERR_CUDA; }
  return WD_OK;
}

template <int NQ, int NSEG, typename TI, int BK>
static wd_status launch_attn_tc(const CUtensorMap& tq, const CUtensorMap& tk0, const CUtensorMap& tv0,
                                const CUtensorMap& tk1, const CUtensorMap& tv1, const tca::Params& p, int batch,
                                int heads, bool cross, cudaStream_t st) {
  using C = tca::Cfg<NQ, NSEG, TI, BK>;
  static bool attr[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 15]) {
    cudaFuncSetAttribute(tca::k_attn_tc<NQ, NSEG, TI, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    attr[dev & 15] = true;
  }
  dim3 grid((p.Lq + tca::BQ * NQ - 1) / (tca::BQ * NQ), heads, batch);
  Trace tr(cross ? KC_ATTN_CROSS : KC_ATTN_SELF, st);
  tca::k_attn_tc<NQ, NSEG, TI, BK><<<grid, C::THREADS, C::SMEM, st>>>(tq, tk0, tv0, tk1, tv1, p);
  return launch_status("attention_tc");
}

// The q/k/v pointers of AttnArgs may point into the middle of a row (the
// fused q|k|v buffer); the tensor maps start at the row's first element that
// is 16-byte aligned (the pointer itself) and use the row stride as extent.
template <typename TI>
static wd_status attention_tc_t(const AttnArgs<TI, bf16>& a, cudaStream_t st) {
  if (a.dh != tca::DH) return attention_simt<TI, bf16>(a, st);
  if (a.n1 <= 0 || (a.k2 && a.n2 <= 0)) { set_error("attention: empty key segment"); return WD_ERR_SHAPE; }
  const int D = a.heads * a.dh;
  auto al = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
  if (!al(a.q) || !al(a.k1) || !al(a.v1) || (a.k2 && (!al(a.k2) || !al(a.v2))) || !al(a.o) || (a.q_rs % 8) ||
      (a.kv1_rs % 8) || (a.kv2_rs % 8) || (a.o_rs % 8)) {
    set_error("attention_tc: operands must be 16-byte aligned with row strides multiple of 8");
    return WD_ERR_ALIGN;
  }
  const CUtensorMapDataType ty =
      std::is_same<TI, f16>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tq, tk0, tv0, tk1, tv1;
  // Each map covers D columns from its own base pointer.
  WD_TRY(make_tmap_3d(&tq, ty, a.q, D, a.Lq, a.batch, a.q_rs, a.q_rs * a.Lq));
  const int64_t b1 = a.kv1_bs ? a.batch : 1;
  // keys per block: the self-attention's (one segment) or 128 (two segments)
  constexpr int BK1 = WD_ATTN_SELF_BK;
  const int bk = a.k2 ? 128 : BK1;
  WD_TRY(make_tmap_3d(&tk0, ty, a.k1, D, a.n1, b1, a.kv1_rs, a.kv1_bs, bk));
  WD_TRY(make_tmap_3d(&tv0, ty, a.v1, D, a.n1, b1, a.kv1_rs, a.kv1_bs, bk));
  tca::Params p{};
  p.Lq = a.Lq;
  p.seg[0] = tca::Seg{a.n1, a.kv1_bs == 0};
  p.o = a.o;
  p.o_rs = a.o_rs;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.dh));
  p.lse = a.k2 ? nullptr : a.lse;
  p.heads = a.heads;
  if (a.k2) {
    const int64_t b2 = a.kv2_bs ? a.batch : 1;
    WD_TRY(make_tmap_3d(&tk1, ty, a.k2, D, a.n2, b2, a.kv2_rs, a.kv2_bs));
    WD_TRY(make_tmap_3d(&tv1, ty, a.v2, D, a.n2, b2, a.kv2_rs, a.kv2_bs));
    p.seg[1] = tca::Seg{a.n2, a.kv2_bs == 0};
    return launch_attn_tc<1, 2, TI, 128>(tq, tk0, tv0, tk1, tv1, p, a.batch, a.heads, a.cross, st);
  }
  return launch_attn_tc<2, 1, TI, BK1>(tq, tk0, tv0, tk0, tv0, p, a.batch, a.heads, a.cross, st);
}

wd_status attention_tc(const AttnArgs<bf16, bf16>& a, cudaStream_t st) { return attention_tc_t<bf16>(a, st); }
wd_status attention_tc(const AttnArgs<f16, bf16>& a, cudaStream_t st) { return attention_tc_t<f16>(a, st); }

}  // namespace wd
