// k_gemm_tc.cu — bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA)
// with the epilogues of the DiT block fused in: bias, bias+GELU, bias then
// gate * (.) added into the fp32 residual stream, fp32 store, IEEE half store
// (cross-attention operands), unpatchify.
//
// C[m, n] = sum_k A[m, k] * B[n, k]: A = activations [M, K], B = a Linear
// weight [N, K]; both K-major, loaded by TMA into 128-byte-swizzled shared
// memory tiles of 64 K-elements.
//
// CTA = 2 + 4 * epi_wg warps, persistent over output tiles of 128 x BN:
//   warp 0     TMA producer (one lane): STAGES-deep ring of (A, B) tiles
//   warp 1     TMEM owner + MMA issuer (one lane): 128 x BN x 16 UMMAs,
//              accumulating in one of two TMEM buffers
//   warps 2..  epilogue, epi_wg warpgroups: each warp reads its 32-lane
//              quarter of the accumulator for its warpgroup's share of the
//              columns (tcgen05.ld), applies the epilogue and stores; they
//              release the TMEM buffer so the next tile's MMAs overlap it.
//              The 2-byte outputs and the residual go out through shared-memory
//              staging tiles and TMA stores / reduce-adds (whole 128-byte rows);
//              fp32 stores and the unpatchify scatter store from registers.
#include "wd_internal.cuh"

#include <cudaTypedefs.h>

namespace wd {
namespace tcg {

constexpr int BM = 128, BK = 64;
// Epilogue warpgroups per mode, each taking an equal share of a tile's columns:
// two for the GELU epilogue (a reciprocal and an exponential per element; with
// e4m3 operands it would outlast the MMAs of a tile on one), one otherwise.
template <int MODE> __host__ __device__ constexpr int epi_wg() { return MODE == EPI_GELU ? 2 : 1; }
template <int MODE> __host__ __device__ constexpr int threads() { return 64 + 128 * epi_wg<MODE>(); }
// Epilogues with a 2-byte output go out through TMA stores: each epilogue warp
// packs 32 rows x 64 columns (one 128-byte row per output row) into a
// 128-byte-swizzled staging tile and one lane stores the box, so global memory
// sees whole 128-byte rows instead of 16-byte pieces of 32 rows.  Staging
// buffers per warp: two with one epilogue warpgroup, one with two.
template <int MODE> __host__ __device__ constexpr bool staged2() {
  return MODE == EPI_STORE || MODE == EPI_GELU || MODE == EPI_STORE_F16;
}
template <int MODE> __host__ __device__ constexpr int stg_bufs() { return epi_wg<MODE>() == 1 ? 2 : 1; }
constexpr int STG2_TILE = 32 * 128;   // bytes of one staging tile: 32 rows x 64 two-byte columns

template <int BN>
struct Cfg {
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr int BAR_BYTES = 256;
  // gated residual: per epilogue warp two 32 x 32 fp32 staging tiles for the TMA reduce-add
  static constexpr int RESID_STAGE_BYTES = 32 * 32 * 4;
  static constexpr int STG_BYTES = 4 * 2 * RESID_STAGE_BYTES;
  // staging bytes in front of the barriers: the residual tiles, or the 2-byte store tiles (32 KB either way)
  __host__ __device__ static constexpr int stg(int mode) {
    return mode == EPI_RESID ? STG_BYTES
                             : ((mode == EPI_STORE || mode == EPI_GELU || mode == EPI_STORE_F16) ? 8 * STG2_TILE : 0);
  }
  static constexpr int smem(int mode) { return 1024 + STAGES * STAGE_BYTES + stg(mode) + BAR_BYTES; }
  static_assert(1024 + STAGES * STAGE_BYTES + STG_BYTES + BAR_BYTES <= 232448, "shared memory budget of one CTA exceeded");
  static_assert(8 * STG2_TILE <= STG_BYTES, "2-byte staging within the residual staging budget");
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 0);
  static constexpr uint32_t IDESC_F8 = idesc_e4m3(BM, BN, 0, 0);
};

// Wait-site ids recorded in the device error word on a timeout.
enum : unsigned { SITE_EMPTY = 0x101, SITE_FULL = 0x102, SITE_TFULL = 0x103, SITE_TEMPTY = 0x104, SITE_DRAIN = 0x105 };

// ------------------------------------------------------------------ epilogue on 32 columns
// One thread = one output row m; columns n .. n+31 come from the accumulator.
// The values before the store: FP8 scales (row scale sm = sa[m], passed in so
// that rows past M need not read it), bias, GELU.
// Pairs of columns go through the packed fp32 instructions (f32x2), which
// round each lane as the scalar ones would.
template <int MODE>
__device__ __forceinline__ void epi_values32(const Epi& ep, float sm, int n, const uint32_t (&r)[32], float (&v)[32]) {
  float2 w[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
  if (ep.sa) {   // FP8 operands: acc * (sa[m] * sb[n])
    const float2 sm2 = make_float2(sm, sm);
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(ep.sb + n + 2 * j));
      w[j] = fmul2(w[j], fmul2(sm2, make_float2(b.x, b.y)));
      w[j + 1] = fmul2(w[j + 1], fmul2(sm2, make_float2(b.z, b.w)));
    }
  }
  if (ep.bias) {
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(ep.bias + n + 2 * j));
      w[j] = fadd2(w[j], make_float2(b.x, b.y));
      w[j + 1] = fadd2(w[j + 1], make_float2(b.z, b.w));
    }
  }
  if constexpr (MODE == EPI_GELU) {
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = gelu_as2(w[j]);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) { v[2 * j] = w[j].x; v[2 * j + 1] = w[j].y; }
}
// 8 values packed as 2-byte elements of the epilogue's output type
template <int MODE>
__device__ __forceinline__ uint4 pack8(const float* v) {
  if constexpr (MODE == EPI_STORE_F16)
    return make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]), pack_f16x2(v[6], v[7]));
  else
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

template <int MODE>
__device__ __forceinline__ void epilogue32(const Epi& ep, int64_t m, int n, const uint32_t (&r)[32]) {
  float v[32];
  epi_values32<MODE>(ep, ep.sa ? ep.sa[m] : 0.f, n, r, v);
  if constexpr (MODE == EPI_STORE || MODE == EPI_GELU) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(ep.out) + m * ep.ldo + n);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dst[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                          pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    }
  } else if constexpr (MODE == EPI_STORE_F16) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<f16*>(ep.out) + m * ep.ldo + n);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dst[j] = make_uint4(pack_f16x2(v[8 * j], v[8 * j + 1]), pack_f16x2(v[8 * j + 2], v[8 * j + 3]),
                          pack_f16x2(v[8 * j + 4], v[8 * j + 5]), pack_f16x2(v[8 * j + 6], v[8 * j + 7]));
    }
  } else if constexpr (MODE == EPI_F32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(ep.out) + m * ep.ldo + n);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else {   // EPI_UNPATCH
    float* out = static_cast<float*>(ep.out);
#pragma unroll
    for (int j = 0; j < 32; ++j) out[unpatch_index(ep, m, n + j)] = v[j];
  }
}

// ------------------------------------------------------------------ kernel
template <int BN, int MODE, bool F8>
__global__ void __launch_bounds__(threads<MODE>(), 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmX, const Epi ep, int M, int N, int K) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  float* stg = reinterpret_cast<float*>(sB + C::STAGES * C::B_BYTES);   // 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES + C::stg(MODE));
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;   // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* tdone = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = N / BN;
  const int m_tiles = (M + BM - 1) / BM;
  const int tiles = m_tiles * n_tiles;
  constexpr int KS = F8 ? 2 * BK : BK;   // K elements per 128-byte stage row
  const int k_iters = (K + KS - 1) / KS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4 * epi_wg<MODE>()); }
    mbar_init(tdone, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;   // per-stage bit masks
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
        for (int k = 0; k < k_iters; ++k) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, SITE_EMPTY)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, k * KS, m0, &full[stage]);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, k * KS, n0, &full[stage]);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      for (int s = 0; s < C::STAGES; ++s)
        if (issued & (1u << s)) mbar_wait(&full[s], (last_par >> s) & 1u, SITE_DRAIN);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      // Shared-memory descriptors as (low, high) halves: the high half is fixed and
      // the start-address field in the low half steps by 16-byte units.
      const uint64_t da0 = sdesc_sw128(smem_u32(sA), 16, 1024), db0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      const uint32_t a_lo0 = static_cast<uint32_t>(da0), b_lo0 = static_cast<uint32_t>(db0);
      const uint32_t d_hi = static_cast<uint32_t>(da0 >> 32);
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, SITE_TEMPTY)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int k = 0; k < k_iters; ++k) {
          if (!mbar_wait(&full[stage], phase, SITE_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_lo = a_lo0 + stage * (C::A_BYTES >> 4), b_lo = b_lo0 + stage * (C::B_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {   // 32 bytes of K per MMA: 16 bf16 or 32 e4m3 elements
            if constexpr (F8)
              umma_ss_f8_lh(d, a_lo + kk * 2, d_hi, b_lo + kk * 2, d_hi, C::IDESC_F8, (k | kk) != 0);
            else
              umma_ss_lh(d, a_lo + kk * 2, d_hi, b_lo + kk * 2, d_hi, C::IDESC, (k | kk) != 0);
          }
          umma_commit(&empty[stage]);   // frees the smem slot once these MMAs have read it
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);       // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Every MMA issued above has completed once tdone flips.
      umma_commit(tdone);
      mbar_wait(tdone, 0, SITE_DRAIN);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue warps
    const int q = warp & 3;   // TMEM lane quarter this warp may access
    constexpr int COLS = BN / epi_wg<MODE>();
    const int c_begin = ((warp - 2) >> 2) * COLS;
    int acc = 0;
    uint32_t acc_phase = 0;
    [[maybe_unused]] uint32_t chunk = 0;   // residual staging tiles used so far (alternating)
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
      if (!mbar_wait_warp(&tfull[acc], acc_phase, SITE_TFULL)) break;
      tc_fence_after();
      const int64_t m = m0 + q * 32 + lane;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      if constexpr (MODE == EPI_RESID) {
        // X[m, n] += g[n] * v through the TMA: this warp's 32 rows x 32 columns
        // go to a 128-byte-swizzled staging tile (row `lane`, 16-byte chunk j
        // at chunk j ^ (lane & 7)), then one lane reduces the tile into X in
        // L2, so no residual load waits in the SM.
        const bool gated = ep.gate_a || ep.gate_b;
        // FP8 row scale of this thread's row, read once per tile (inside the column loop the
        // compiler cannot keep it across the staging-tile stores)
        const float rs = (ep.sa && m < M) ? ep.sa[m] : 0.f;
#pragma unroll 1
        for (int c = c_begin; c < c_begin + COLS; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          float* tile = stg + ((warp - 2) * 2 + (chunk & 1)) * (32 * 32);
          if (lane == 0) bulk_wait_group_read<1>();   // the reduce that last read this tile is done with it
          __syncwarp();
          tmem_wait_ld();
          float4* row = reinterpret_cast<float4*>(tile + lane * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int n = n0 + c + 4 * j;
            float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
            if (gated) {
              const float4 ga = ep.gate_a ? __ldg(reinterpret_cast<const float4*>(ep.gate_a + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
              const float4 gb = ep.gate_b ? __ldg(reinterpret_cast<const float4*>(ep.gate_b + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
              g = make_float4(ga.x + gb.x, ga.y + gb.y, ga.z + gb.z, ga.w + gb.w);
            }
            const float4 bb = ep.bias ? __ldg(reinterpret_cast<const float4*>(ep.bias + n)) : make_float4(0.f, 0.f, 0.f, 0.f);
            float4 a = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                   __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
            if (ep.sa) {   // FP8 operands: acc * (sa[m] * sb[n])
              const float4 sb = __ldg(reinterpret_cast<const float4*>(ep.sb + n));
              a.x *= rs * sb.x; a.y *= rs * sb.y; a.z *= rs * sb.z; a.w *= rs * sb.w;
            }
            row[j ^ (lane & 7)] = make_float4(g.x * (a.x + bb.x), g.y * (a.y + bb.y), g.z * (a.z + bb.z), g.w * (a.w + bb.w));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && m0 + q * 32 < M) {   // rows past M inside the box are skipped by the TMA
            tma_reduce_add_2d(tile, &tmX, n0 + c, m0 + q * 32);
            bulk_commit_group();
          }
          ++chunk;
        }
      } else if constexpr (staged2<MODE>() && COLS % 64 == 0) {
        // 64 columns at a time: values packed into this warp's staging tile
        // (row `lane`, 16-byte chunk j at chunk j ^ (lane & 7)), then one lane
        // stores the 32 x 64 box; rows past M inside the box are clipped by the TMA.
        constexpr int NB = stg_bufs<MODE>();
        const float sm = (ep.sa && m < M) ? ep.sa[m] : 0.f;
#pragma unroll 1
        for (int c = c_begin; c < c_begin + COLS; c += 64) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + c, r0);
          tmem_ld32(tbase + c + 32, r1);
          uint8_t* tile = reinterpret_cast<uint8_t*>(stg) + ((warp - 2) * NB + (chunk % NB)) * STG2_TILE;
          if (lane == 0) bulk_wait_group_read<NB - 1>();   // the store that last read this tile is done with it
          __syncwarp();
          tmem_wait_ld();
          uint4* row = reinterpret_cast<uint4*>(tile + lane * 128);
          float v[32];
          epi_values32<MODE>(ep, sm, n0 + c, r0, v);
#pragma unroll
          for (int j = 0; j < 4; ++j) row[j ^ (lane & 7)] = pack8<MODE>(v + 8 * j);
          epi_values32<MODE>(ep, sm, n0 + c + 32, r1, v);
#pragma unroll
          for (int j = 0; j < 4; ++j) row[(4 + j) ^ (lane & 7)] = pack8<MODE>(v + 8 * j);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && m0 + q * 32 < M) {
            tma_store_2d(tile, &tmX, n0 + c, m0 + q * 32);
            bulk_commit_group();
          }
          ++chunk;
        }
      } else {
#pragma unroll 1
        for (int c = c_begin; c < c_begin + COLS; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tmem_wait_ld();
          if (m < M) epilogue32<MODE>(ep, m, n0 + c, r);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if ((MODE == EPI_RESID || (staged2<MODE>() && COLS % 64 == 0)) && lane == 0)
      bulk_wait_group<0>();   // reductions and stores performed before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace tcg

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D tensor map over a row-major [rows, cols] matrix of bf16 (or, with
// one_byte, e4m3 codes as uint8) with row stride `ld` elements; box =
// box_cols x box_rows, 128-byte swizzle.
static wd_status make_tmap_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                                int box_cols, int box_rows, bool one_byte = false) {
  auto fn = encode_fn();
  if (!fn) { set_error("cuTensorMapEncodeTiled unavailable"); return WD_ERR_CUDA; }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * (one_byte ? 1 : 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { set_error("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r)); return WD_ERR_CUDA; }
  return WD_OK;
}

static int sm_count() {
  static int cnt[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!cnt[dev & 15]) cudaDeviceGetAttribute(&cnt[dev & 15], cudaDevAttrMultiProcessorCount, dev);
  return cnt[dev & 15];
}

// 2D fp32 tensor map over the residual stream [rows, cols], box_cols x box_rows,
// 128-byte swizzle (box_cols = 32: one 128-byte row per box row).
static wd_status make_tmap_f32(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_cols,
                               int box_rows) {
  auto fn = encode_fn();
  if (!fn) { set_error("cuTensorMapEncodeTiled unavailable"); return WD_ERR_CUDA; }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { set_error("cuTensorMapEncodeTiled (f32) failed (%d)", static_cast<int>(r)); return WD_ERR_CUDA; }
  return WD_OK;
}

// 2D tensor map over a 2-byte output [rows, cols] (bf16, or IEEE half), row
// stride ld elements; box 64 x 32 (one 128-byte row per box row), 128-byte swizzle.
static wd_status make_tmap_2b(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, bool half) {
  auto fn = encode_fn();
  if (!fn) { set_error("cuTensorMapEncodeTiled unavailable"); return WD_ERR_CUDA; }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, half ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { set_error("cuTensorMapEncodeTiled (2-byte out) failed (%d)", static_cast<int>(r)); return WD_ERR_CUDA; }
  return WD_OK;
}

template <int BN, int MODE, bool F8 = false>
static wd_status launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const Epi& ep, int M, int N, int K,
                           cudaStream_t st) {
  using C = tcg::Cfg<BN>;
  static bool attr[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr[dev & 15]) {
    cudaFuncSetAttribute(tcg::k_gemm_tc<BN, MODE, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::smem(MODE));
    attr[dev & 15] = true;
  }
  const int tiles = ((M + tcg::BM - 1) / tcg::BM) * (N / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  CUtensorMap tx = ta;   // the residual (fp32) or 2-byte output map of the TMA epilogues, else unused
  if (MODE == EPI_RESID) WD_TRY(make_tmap_f32(&tx, ep.out, M, N, ep.ldo, 32, 32));
  if (tcg::staged2<MODE>() && (BN / tcg::epi_wg<MODE>()) % 64 == 0)
    WD_TRY(make_tmap_2b(&tx, ep.out, M, N, ep.ldo, MODE == EPI_STORE_F16));
  Trace tr(KC_GEMM, st);
  tcg::k_gemm_tc<BN, MODE, F8><<<grid, tcg::threads<MODE>(), C::smem(MODE), st>>>(ta, tb, tx, ep, M, N, K);
  return launch_status("gemm_tc");
}

template <int BN>
static wd_status dispatch_mode(int mode, const CUtensorMap& ta, const CUtensorMap& tb, const Epi& ep, int M, int N,
                               int K, cudaStream_t st) {
  switch (mode) {
    case EPI_STORE: return launch_tc<BN, EPI_STORE>(ta, tb, ep, M, N, K, st);
    case EPI_GELU: return launch_tc<BN, EPI_GELU>(ta, tb, ep, M, N, K, st);
    case EPI_F32: return launch_tc<BN, EPI_F32>(ta, tb, ep, M, N, K, st);
    case EPI_RESID: return launch_tc<BN, EPI_RESID>(ta, tb, ep, M, N, K, st);
    case EPI_UNPATCH: return launch_tc<BN, EPI_UNPATCH>(ta, tb, ep, M, N, K, st);
    case EPI_STORE_F16: return launch_tc<BN, EPI_STORE_F16>(ta, tb, ep, M, N, K, st);
  }
  set_error("gemm_tc: bad epilogue %d", mode);
  return WD_ERR_ARG;
}

wd_status gemm_tc(int M, int N, int K, const bf16* A, int64_t lda, const bf16* B, int64_t ldb, int mode,
                  const Epi& ep, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) { set_error("gemm: empty shape %d x %d x %d", M, N, K); return WD_ERR_SHAPE; }
  // TMA rules: 16-byte aligned base and row strides.
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) & 15u) {
    set_error("gemm_tc: operands must be 16-byte aligned");
    return WD_ERR_ALIGN;
  }
  if ((lda % 8) || (ldb % 8) || (K % 8)) {
    set_error("gemm_tc: K=%d, lda=%lld, ldb=%lld must be multiples of 8", K, (long long)lda, (long long)ldb);
    return WD_ERR_SHAPE;
  }
  if (N % 64) { set_error("gemm_tc: N=%d must be a multiple of 64", N); return WD_ERR_SHAPE; }
  if (mode != EPI_UNPATCH && (ep.ldo % 8 || (reinterpret_cast<uintptr_t>(ep.out) & 15u))) {
    set_error("gemm_tc: output must be 16-byte aligned with ldo %% 8 == 0");
    return WD_ERR_ALIGN;
  }
  const int BN = (N % 256 == 0) ? 256 : ((N % 128 == 0) ? 128 : 64);
  CUtensorMap ta, tb;
  WD_TRY(make_tmap_bf16(&ta, A, M, K, lda, tcg::BK, tcg::BM));
  WD_TRY(make_tmap_bf16(&tb, B, N, K, ldb, tcg::BK, BN));
  switch (BN) {
    case 256: return dispatch_mode<256>(mode, ta, tb, ep, M, N, K, st);
    case 128: return dispatch_mode<128>(mode, ta, tb, ep, M, N, K, st);
    default: return dispatch_mode<64>(mode, ta, tb, ep, M, N, K, st);
  }
}

// e4m3 operands: N a multiple of 256 (one tile width), K and the row strides
// multiples of 16 bytes; the block's GEMMs all have that shape.
wd_status gemm_tc_fp8(int M, int N, int K, const uint8_t* A, int64_t lda, const uint8_t* B, int64_t ldb, int mode,
                      const Epi& ep, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) { set_error("gemm_fp8: empty shape %d x %d x %d", M, N, K); return WD_ERR_SHAPE; }
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) & 15u) {
    set_error("gemm_fp8: operands must be 16-byte aligned");
    return WD_ERR_ALIGN;
  }
  if ((lda % 16) || (ldb % 16) || (K % 16)) {
    set_error("gemm_fp8: K=%d, lda=%lld, ldb=%lld must be multiples of 16", K, (long long)lda, (long long)ldb);
    return WD_ERR_SHAPE;
  }
  if (N % 256) { set_error("gemm_fp8: N=%d must be a multiple of 256", N); return WD_ERR_SHAPE; }
  if (!ep.sa || !ep.sb) { set_error("gemm_fp8: row and column scales are required"); return WD_ERR_ARG; }
  if (ep.ldo % 8 || (reinterpret_cast<uintptr_t>(ep.out) & 15u)) {
    set_error("gemm_fp8: output must be 16-byte aligned with ldo %% 8 == 0");
    return WD_ERR_ALIGN;
  }
  CUtensorMap ta, tb;
  WD_TRY(make_tmap_bf16(&ta, A, M, K, lda, 2 * tcg::BK, tcg::BM, true));
  WD_TRY(make_tmap_bf16(&tb, B, N, K, ldb, 2 * tcg::BK, 256, true));
  switch (mode) {
    case EPI_STORE: return launch_tc<256, EPI_STORE, true>(ta, tb, ep, M, N, K, st);
    case EPI_GELU: return launch_tc<256, EPI_GELU, true>(ta, tb, ep, M, N, K, st);
    case EPI_F32: return launch_tc<256, EPI_F32, true>(ta, tb, ep, M, N, K, st);
    case EPI_RESID: return launch_tc<256, EPI_RESID, true>(ta, tb, ep, M, N, K, st);
    case EPI_STORE_F16: return launch_tc<256, EPI_STORE_F16, true>(ta, tb, ep, M, N, K, st);
  }
  set_error("gemm_fp8: bad epilogue %d", mode);
  return WD_ERR_ARG;
}

}  // namespace wd
