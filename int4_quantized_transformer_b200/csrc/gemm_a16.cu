// gemm_a16.cu -- the quantized linear layer with FP16 activations, W8A16 and
// W4A16 (ZeroQuant, arXiv 2206.01861; summary page "ZeroQuant: Efficient and
// Affordable Post-Training Quantization for Large-Scale Transformers",
// sections "Main Quantitative Results" (W8A16) and "INT4/INT8 Mixed-Precision
// Quantization" (W4/8A16, and GPT-NeoX's self-attention input kept in FP16
// while its weights stay quantized)).
//
//   acc[t,o] = sum_k x[t,k] * q[o,k]            fp16 x integer code, fp32 sum
//   Y[t,o]   = fp16( fp32(acc[t,o] * s_grp[group(o)]) + f32(bias[o]) )
//
// A group's scale is constant along every row of W that it covers, so the
// dequantized weight q*S contributes S * sum_k x*q: the codes enter the
// tensor core as exact fp16 integers and the scale is applied once per
// output, in the epilogue.
//
// One persistent CTA per SM walks 128 x BN output tiles (token rows on the
// MMA M side); with ZQ_OPT_CTA_PAIR = 2 a CTA pair (cta_group::2) walks
// 256 x BN units instead, each CTA widening half of the weight tile (built
// and tested, but measured slower, so never chosen automatically).  Warp
// roles:
//   warp 0       TMA producer: per 64-element K slice, the fp16 activation
//                tile (128 rows, 128-byte swizzle, the MMA's K-major layout)
//                and the codes of BN weight rows (plain rows);
//   warp 1       MMA issuer: tcgen05.mma kind::f16, M = 128, N = BN, K = 16,
//                into one of two fp32 TMEM accumulator buffers, so that the
//                epilogue of one tile overlaps the mainloop of the next;
//   warps 2-9    epilogue: TMEM -> registers, scale and bias, fp16, TMA
//                stores of 32 x 32 blocks;
//   warps 10-13  widen the codes to fp16 in the 128-byte-swizzled K-major
//                layout.  An int8 or int4 code c becomes the fp16 bit pattern
//                0x6400 + (c + bias) -- the number 1024 + c + bias, exact --
//                and one packed fp16 subtraction of 1024 + bias leaves c.
// Every wait is bounded (see zq_ptx.cuh): a stuck pipeline records where it
// gave up in the device status word and the CTA leaves.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "zq_internal.h"
#include "zq_ptx.cuh"

namespace zq {
namespace {

constexpr int kBM = 128;      // token rows of a tile = TMEM lanes
constexpr int kKE = 64;       // fp16 elements per K slice: one 128-byte swizzle row
constexpr int kUmmaK = 16;    // K of one kind::f16 MMA (32 bytes)
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant
constexpr int kCvtWarps = 4;
constexpr int kBudget = 223 * 1024;

constexpr int tmem_cols_for(int v) {
  int p = 32;
  while (p < v) p *= 2;
  return p;
}

template <int BN_, bool W4_, bool PAIR_, bool PRE_ = false>
struct A16Cfg {
  static constexpr int BN = BN_;
  static constexpr bool W4 = W4_;
  // PRE: the weights were widened to fp16 codes before the launch
  // (widen_a16_kernel) and reach shared memory by TMA like the activations;
  // the widening warps then have nothing to do.
  static constexpr bool PRE = PRE_;
  static_assert(!PRE || !W4, "pre-widened weights are fp16 whatever their code width");
  // CTA pair (cta_group::2): a 256 x BN tile per pair; each CTA holds 128
  // token rows of A, widens BN/2 weight rows of B, and keeps 128 rows of D.
  static constexpr bool PAIR = PAIR_;
  static constexpr int TILE_M = PAIR ? 2 * kBM : kBM;  // token rows of a unit
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;    // weight rows this CTA widens
  static constexpr int A_BYTES = kBM * 128;            // fp16 activations of one slice
  static constexpr int B_BYTES = B_ROWS * 128;         // widened weights of one slice
  static constexpr int CODE_ROW = W4 ? kKE / 2 : kKE;  // code bytes per weight row and slice
  static constexpr int P_BYTES = PRE ? 0 : B_ROWS * CODE_ROW;  // codes as stored in memory
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + P_BYTES;
  static constexpr int EPI_COLS = BN / 2;              // columns of one epilogue warp
  static constexpr int STG_BYTES = 32 * 32 * 2;        // one 32 x 32 fp16 output block
  static constexpr int FREE = kBudget - kEpiWarps * STG_BYTES - kEpiWarps * EPI_COLS * 8;
  static constexpr int STAGES_RAW = FREE / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int TMEM_COLS = tmem_cols_for(2 * BN);
  static constexpr int NUM_WARPS = 2 + kEpiWarps + kCvtWarps;
  static constexpr int NUM_THREADS = 32 * NUM_WARPS;
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_P = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_EPI = OFF_P + STAGES * P_BYTES;
  static constexpr int EPI_BYTES = kEpiWarps * EPI_COLS * 2 * 4;
  static constexpr int OFF_STG = ((OFF_EPI + EPI_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_BAR = OFF_STG + kEpiWarps * STG_BYTES;
  static constexpr int NUM_BARS = 4 * STAGES + 4 + 1;
  static constexpr int READY_ARRIVALS = PAIR ? 2 * kCvtWarps : kCvtWarps;
  static constexpr int EPI_ARRIVALS = PAIR ? 2 * kEpiWarps : kEpiWarps;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "MMA N and the epilogue's 64-column steps");
  static_assert(B_ROWS % 16 == 0, "widening steps of 16 rows keep each row's swizzle phase");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(P_BYTES % 128 == 0, "TMA destination alignment");
  static_assert(!PRE || B_ROWS <= 256, "one TMA box of weight rows");
  static_assert(EPI_COLS <= 128, "epilogue prefetch holds at most four columns per lane");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(TMEM_COLS <= 512, "TMEM accumulators");
};

struct A16Params {
  const float* s_grp;
  const __half* bias;
  float* acc_dbg;
  int* status;
  int T, N, K, g;
  int m_tiles, n_tiles, k_blocks, num_units;
};

// group(o) = floor(o * g / N), 32-bit whenever o * g fits.
__device__ __forceinline__ int a16_group_of(int o, int N, int g) {
  const unsigned long long prod = static_cast<unsigned long long>(o) * static_cast<unsigned>(g);
  if (prod < (1ull << 32)) return static_cast<int>(static_cast<unsigned>(prod) / static_cast<unsigned>(N));
  return static_cast<int>(prod / static_cast<unsigned>(N));
}

// Warp-uniform bounded wait (lane 0 polls; the verdict is broadcast).
__device__ __forceinline__ bool a16_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              int* status, int site) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status, site) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Four int8 codes (one 32-bit word, k order) -> two fp16x2 words.  Flipping
// the sign bit of each byte gives c + 128 in 0..255; placed under the fp16
// exponent byte 0x64 it is the number 1024 + c + 128 (exact, unit spacing in
// [1024, 2048)), and subtracting 1152 leaves c exactly.
__device__ __forceinline__ void widen4_i8(uint32_t w, uint32_t& h01, uint32_t& h23) {
  const uint32_t u = w ^ 0x80808080u;
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  uint32_t a = __byte_perm(u, 0x64646464u, 0x5140);  // bytes: c0', 0x64, c1', 0x64
  uint32_t b = __byte_perm(u, 0x64646464u, 0x7362);  // bytes: c2', 0x64, c3', 0x64
  __half2 ha = __hsub2(*reinterpret_cast<__half2*>(&a), off);
  __half2 hb = __hsub2(*reinterpret_cast<__half2*>(&b), off);
  h01 = *reinterpret_cast<uint32_t*>(&ha);
  h23 = *reinterpret_cast<uint32_t*>(&hb);
}

// Eight int4 codes of one 32-bit word (byte i: k = i in the low nibble, k = 4
// + i in the high nibble) -> four fp16x2 words in k order.  Flipping each
// nibble's sign bit gives c + 8 in 0..15; under 0x64 that is 1024 + c + 8,
// and subtracting 1032 leaves c.
__device__ __forceinline__ void widen8_i4(uint32_t w, uint32_t (&h)[4]) {
  const uint32_t u = w ^ 0x88888888u;
  const uint32_t lo = u & 0x0F0F0F0Fu;         // k = 0..3
  const uint32_t hi = (u >> 4) & 0x0F0F0F0Fu;  // k = 4..7
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  uint32_t v[4] = {__byte_perm(lo, 0x64646464u, 0x5140), __byte_perm(lo, 0x64646464u, 0x7362),
                   __byte_perm(hi, 0x64646464u, 0x5140), __byte_perm(hi, 0x64646464u, 0x7362)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 x = __hsub2(*reinterpret_cast<__half2*>(&v[i]), off);
    h[i] = *reinterpret_cast<uint32_t*>(&x);
  }
}

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    gemm_a16_kernel(const __grid_constant__ CUtensorMap map_x,
                    const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_y, const A16Params p) {
  constexpr int BN = C::BN;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sP = smem + C::OFF_P;
  float* sEpi = reinterpret_cast<float*>(smem + C::OFF_EPI);
  uint8_t* sStg = smem + C::OFF_STG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // Single CTA: full = activations + codes landed.  Pair: full (the leader's)
  // counts both CTAs' activation tiles, pfull this CTA's codes.
  uint64_t* full_bar = bars;                  // [STAGES]
  uint64_t* ready_bar = bars + STAGES;        // [STAGES] widened weights written (leader's, pair)
  uint64_t* empty_bar = bars + 2 * STAGES;    // [STAGES] the MMAs reading the stage are done
  uint64_t* pfull_bar = bars + 3 * STAGES;    // [STAGES] pair: this CTA's codes landed
  uint64_t* tfull_bar = bars + 4 * STAGES;    // [2] accumulator buffer complete
  uint64_t* tempty_bar = tfull_bar + 2;       // [2] accumulator buffer drained
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  // a pair works on one unit at a time; crank 0 (the leader) issues the MMAs
  const uint32_t crank = C::PAIR ? cluster_ctarank() : 0u;
  const int unit0 = C::PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int ustep = C::PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&ready_bar[s], C::READY_ARRIVALS);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&pfull_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], C::EPI_ARRIVALS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_w);
    tma_prefetch_desc(&map_y);
  }
  if (warp == 1) {
    if constexpr (C::PAIR) {
      tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (C::PAIR) cluster_sync_all();  // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // Nothing above touches global memory; what follows may read what the
  // previous kernel of the stream wrote.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_last();
      const uint64_t pol_w = l2_policy_evict_normal();
      constexpr uint32_t bytes = static_cast<uint32_t>(C::A_BYTES + C::P_BYTES);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[STAGES];
      for (int s = 0; s < STAGES; ++s) fills[s] = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.num_units; u += ustep) {
        const int m = u % p.m_tiles, n = u / p.m_tiles;
        const int act_row = m * C::TILE_M + static_cast<int>(crank) * kBM;
        const int w_row = n * BN + static_cast<int>(crank) * C::B_ROWS;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.status, 21)) {
            ok = false;
            break;
          }
          // slices past K (and rows past T or N) read the TMA's zero fill
          if constexpr (C::PRE) {
            // activations and fp16 weight rows, both in the MMA's layout; for
            // a pair, both CTAs' tiles complete on the leader's full barrier
            if constexpr (C::PAIR) {
              const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
              if (crank == 0)
                mbar_arrive_expect_tx(&full_bar[stage], 2u * (C::A_BYTES + C::B_BYTES));
              tma_load_2d_pair(sA + stage * C::A_BYTES, &map_x, fb, kb * kKE, act_row, pol_x);
              tma_load_2d_pair(sB + stage * C::B_BYTES, &map_w, fb, kb * kKE, w_row, pol_w);
            } else {
              mbar_arrive_expect_tx(&full_bar[stage], C::A_BYTES + C::B_BYTES);
              tma_load_2d(sA + stage * C::A_BYTES, &map_x, &full_bar[stage], kb * kKE, act_row,
                          pol_x);
              tma_load_2d(sB + stage * C::B_BYTES, &map_w, &full_bar[stage], kb * kKE, w_row,
                          pol_w);
            }
          } else if constexpr (C::PAIR) {
            // both CTAs' activation tiles complete on the leader's full
            // barrier (the MMA reads them); this CTA's codes on its own
            // pfull barrier (its widening warps read them)
            if (crank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2u * C::A_BYTES);
            tma_load_2d_pair(sA + stage * C::A_BYTES, &map_x,
                             mapa_shared(smem_u32(&full_bar[stage]), 0), kb * kKE, act_row, pol_x);
            mbar_arrive_expect_tx(&pfull_bar[stage], static_cast<uint32_t>(C::P_BYTES));
            tma_load_2d(sP + stage * C::P_BYTES, &map_w, &pfull_bar[stage], kb * C::CODE_ROW, w_row,
                        pol_w);
          } else {
            mbar_arrive_expect_tx(&full_bar[stage], bytes);
            tma_load_2d(sA + stage * C::A_BYTES, &map_x, &full_bar[stage], kb * kKE, act_row, pol_x);
            tma_load_2d(sP + stage * C::P_BYTES, &map_w, &full_bar[stage], kb * C::CODE_ROW, w_row,
                        pol_w);
          }
          ++fills[stage];
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every copy issued lands before the CTA may exit (for a pair, the
      // leader's full barriers count both CTAs' activation copies; the
      // follower exits only after the final cluster barrier)
      int no_abort = 0;
      if (!C::PAIR || crank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (fills[s]) mbar_wait(&full_bar[s], (fills[s] - 1) & 1, &no_abort, p.status, 22);
      if (C::PAIR && !C::PRE)
        for (int s = 0; s < STAGES; ++s)
          if (fills[s]) mbar_wait(&pfull_bar[s], (fills[s] - 1) & 1, &no_abort, p.status, 28);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0 && (!C::PAIR || crank == 0)) {
      constexpr uint32_t idesc = make_idesc_f16(C::TILE_M, BN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t tphase = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.num_units; u += ustep) {
        if (!mbar_wait(&tempty_bar[buf], tphase ^ 1, abort_flag, p.status, 23)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          // the widening warps arrive only after the stage's codes landed
          // (single CTA: with the activations, on the same barrier); a pair
          // also waits for both CTAs' activation tiles
          if ((!C::PRE && !mbar_wait(&ready_bar[stage], phase, abort_flag, p.status, 24)) ||
              ((C::PAIR || C::PRE) && !mbar_wait(&full_bar[stage], phase, abort_flag, p.status, 29))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = make_sw128_desc(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t db = make_sw128_desc(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < kKE / kUmmaK; ++k) {  // start address + k*32 bytes (>>4 = 2k)
            if constexpr (C::PAIR)
              mma_f16_pair(d_tmem, da + static_cast<uint64_t>(2 * k),
                           db + static_cast<uint64_t>(2 * k), idesc, (kb > 0 || k > 0) ? 1u : 0u);
            else
              mma_f16(d_tmem, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k),
                      idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          if constexpr (C::PAIR)
            mma_commit_pair_mc(&empty_bar[stage], 0x3);
          else
            mma_commit(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if constexpr (C::PAIR)
          mma_commit_pair_mc(&tfull_bar[buf], 0x3);
        else
          mma_commit(&tfull_bar[buf]);
        if (++buf == 2) {
          buf = 0;
          tphase ^= 1;
        }
      }
      // every MMA issued completes before TMEM is released
      if constexpr (C::PAIR)
        mma_commit_pair_mc(drain_bar, 0x1);
      else
        mma_commit(drain_bar);
      int no_abort = 0;
      mbar_wait(drain_bar, 0, &no_abort, p.status, 25);
    }
  } else if (warp < 2 + kEpiWarps) {
    // ------------------------------------------------------ epilogue
    const int ew = warp - 2;    // 0..7
    const int quad = warp & 3;  // the TMEM lane quadrant this warp may read
    const int half = ew >> 2;   // which half of the tile's columns
    const int row_in_tile = quad * 32 + lane;
    const int cb = half * C::EPI_COLS;
    const int ce = cb + C::EPI_COLS;
    float* colv = sEpi + ew * (2 * C::EPI_COLS) - cb;  // scale and bias of columns [cb, ce)
    float* colb = colv + C::EPI_COLS;
    uint8_t* stg = sStg + ew * C::STG_BYTES;
    constexpr int PCOLS = C::EPI_COLS / 32;
    int buf = 0;
    uint32_t tphase = 0;
    // a unit's scales and bias are loaded one unit ahead (lane l holds
    // columns cb + l + 32 i), so their latency overlaps the previous unit
    float n_cv[PCOLS];
    __half n_cb[PCOLS];
    auto fetch = [&](int u) {
#pragma unroll
      for (int i = 0; i < PCOLS; ++i) {
        n_cv[i] = 0.0f;
        n_cb[i] = __float2half_rn(0.0f);
      }
      if (u >= p.num_units) return;
      const int n = u / p.m_tiles;
#pragma unroll
      for (int i = 0; i < PCOLS; ++i) {
        const int o = n * BN + cb + lane + 32 * i;
        if (o < p.N) {
          n_cv[i] = __ldg(p.s_grp + a16_group_of(o, p.N, p.g));
          if (p.bias) n_cb[i] = p.bias[o];
        }
      }
    };
    fetch(unit0);
    for (int u = unit0; u < p.num_units; u += ustep) {
      const int m = u % p.m_tiles, n = u / p.m_tiles;
#pragma unroll
      for (int i = 0; i < PCOLS; ++i) {
        colv[cb + lane + 32 * i] = n_cv[i];
        colb[cb + lane + 32 * i] = __half2float(n_cb[i]);
      }
      __syncwarp();
      if (!a16_wait_warp(&tfull_bar[buf], tphase, abort_flag, p.status, 26)) break;
      tc_fence_after();
      fetch(u + ustep);
      const int tok = m * C::TILE_M + static_cast<int>(crank) * kBM + row_in_tile;
      const int row0 = m * C::TILE_M + static_cast<int>(crank) * kBM + quad * 32;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * BN);

      // 32 accumulator columns -> 16 packed fp16 pairs (and the raw sums)
      auto dequant = [&](const uint32_t (&acc)[32], int c0, uint32_t (&h)[16]) {
        const int o0 = n * BN + c0;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float v0 = __fadd_rn(__fmul_rn(__uint_as_float(acc[j]), colv[c0 + j]), colb[c0 + j]);
          const float v1 =
              __fadd_rn(__fmul_rn(__uint_as_float(acc[j + 1]), colv[c0 + j + 1]), colb[c0 + j + 1]);
          const __half2 hv = __floats2half2_rn(v0, v1);
          h[j / 2] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        if (p.acc_dbg && tok < p.T && o0 < p.N) {
          float* arow = p.acc_dbg + static_cast<size_t>(tok) * p.N + o0;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (o0 + 4 * q < p.N)  // N % 8 == 0, so 4-column chunks are all in or all out
              reinterpret_cast<uint4*>(arow)[q] =
                  make_uint4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
      };
      // the warp's 32 rows x 32 columns leave as one TMA store (rows past T
      // and columns past N are clipped by the TMA unit)
      auto store = [&](const uint32_t (&h)[16], int c0) {
        const int o0 = n * BN + c0;
        if (o0 < p.N && row0 < p.T) {  // warp-uniform
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
          const int sw = (lane >> 1) & 3;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(stg + lane * 64 + ((q ^ sw) << 4)) =
                make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_y, stg, o0, row0);
            bulk_commit_group();
          }
        }
      };
#pragma unroll 1
      for (int c0 = cb; c0 < ce; c0 += 64) {
        uint32_t a0[32], a1[32];
        tmem_ld_32x32b_x32(t_row + c0, a0);
        tmem_ld_32x32b_x32(t_row + c0 + 32, a1);
        tmem_ld_wait();
        uint32_t h[16];
        dequant(a0, c0, h);
        store(h, c0);
        dequant(a1, c0 + 32, h);
        store(h, c0 + 32);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (C::PAIR)
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
        else
          mbar_arrive(&tempty_bar[buf]);
      }
      if (++buf == 2) {
        buf = 0;
        tphase ^= 1;
      }
      __syncwarp();
    }
  } else if constexpr (!C::PRE) {
    // ------------------------------------------------------ widen the codes
    // Thread ut writes 16-byte chunk j = ut % 8 (eight k) of rows
    // r = ut / 8 + 16 i; stepping 16 rows keeps r % 8, so each thread's
    // swizzled chunk position is fixed.
    const int ut = threadIdx.x - 32 * (2 + kEpiWarps);  // 0..127
    const int r0 = ut >> 3, j = ut & 7;
    const int src0 = r0 * C::CODE_ROW + j * (C::CODE_ROW / 8);
    const int dst0 = r0 * 128 + ((j ^ (r0 & 7)) << 4);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int u = unit0; ok && u < p.num_units; u += ustep) {
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        if (!a16_wait_warp(C::PAIR ? &pfull_bar[stage] : &full_bar[stage], phase, abort_flag,
                           p.status, 27)) {
          ok = false;
          break;
        }
        const uint8_t* src = sP + stage * C::P_BYTES + src0;
        uint8_t* dst = sB + stage * C::B_BYTES + dst0;
#pragma unroll 4
        for (int i = 0; i < C::B_ROWS / 16; ++i) {
          uint4 o;
          if constexpr (C::W4) {
            uint32_t h[4];
            widen8_i4(*reinterpret_cast<const uint32_t*>(src + i * 16 * C::CODE_ROW), h);
            o = make_uint4(h[0], h[1], h[2], h[3]);
          } else {
            const uint2 w = *reinterpret_cast<const uint2*>(src + i * 16 * C::CODE_ROW);
            widen4_i8(w.x, o.x, o.y);
            widen4_i8(w.y, o.z, o.w);
          }
          *reinterpret_cast<uint4*>(dst + i * 16 * 128) = o;
        }
        fence_proxy_async_smem();  // generic-proxy writes, read by the tensor core
        __syncwarp();
        if (lane == 0) {
          if constexpr (C::PAIR)
            mbar_arrive_cluster(mapa_shared(smem_u32(&ready_bar[stage]), 0));
          else
            mbar_arrive(&ready_bar[stage]);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }

  __syncwarp();
  if (warp >= 2 && warp < 2 + kEpiWarps && lane == 0) bulk_wait_group0();
  tc_fence_before();
  __syncthreads();
  if constexpr (C::PAIR) cluster_sync_all();  // no CTA leaves while its pair may still signal it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (C::PAIR)
      tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Codes widened once per call to exact fp16 integers [N][K] (the same bit
// construction as the widening warps: the code, sign bit flipped, under the
// exponent byte 0x64, minus 1024 + 128 or 1024 + 8).  HBM-bound: the codes
// are read once and 2*N*K bytes written; the GEMM then reads the fp16 rows
// by TMA, so no tile widens them again.
template <bool W4>
__global__ void __launch_bounds__(256)
    widen_a16_kernel(const uint4* __restrict__ codes, uint4* __restrict__ wide, size_t n16) {
  // the codes may be written by the previous kernel of the stream
  grid_dependency_wait();
  grid_launch_dependents();
  auto one = [&](uint4 w, size_t i) {
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    if constexpr (W4) {  // 32 codes -> 64 bytes
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t h[4];
        widen8_i4(in[m], h);
        wide[4 * i + m] = make_uint4(h[0], h[1], h[2], h[3]);
      }
    } else {  // 16 codes -> 32 bytes
      uint32_t h[8];
#pragma unroll
      for (int m = 0; m < 4; ++m) widen4_i8(in[m], h[2 * m], h[2 * m + 1]);
      wide[2 * i] = make_uint4(h[0], h[1], h[2], h[3]);
      wide[2 * i + 1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
  };
  // four 16-byte loads in flight per thread, so the pass runs at the HBM rate
  constexpr int U = 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  for (; i + (U - 1) * stride < n16; i += U * stride) {
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) w[u] = __ldcs(codes + i + u * stride);
#pragma unroll
    for (int u = 0; u < U; ++u) one(w[u], i + u * stride);
  }
  for (; i < n16; i += stride) one(__ldcs(codes + i), i);
}

// ------------------------------------------------------------------ host

// From this many tokens the codes are widened once per call (widen_a16_kernel)
// and the GEMM reads fp16 weights by TMA; below it the tiles widen them.
constexpr int kA16WidenMinTokens = 1024;

struct A16Plan {
  int bn, m_tiles, n_tiles, k_blocks, units;
  bool pair;
  double cost;
};

// Wave-aware cost in MMA cycles: a 128 x BN x 64 fp16 block takes about
// 2*BN cycles; a fixed charge per tile covers its epilogue tail.  A CTA pair
// does a 256-row unit in the time a single CTA does a 128-row one, with
// half as many pair slots as SMs.
A16Plan plan_a16(int T, int N, int K, int sms, int forced_bn, bool pair) {
  A16Plan best{};
  best.cost = 1e30;
  const int cands[2] = {256, 128};
  const int slots = pair ? sms / 2 : sms;
  for (int bn : cands) {
    if (forced_bn && bn != forced_bn) continue;
    A16Plan p{};
    p.bn = bn;
    p.pair = pair;
    p.m_tiles = (T + (pair ? 2 * kBM : kBM) - 1) / (pair ? 2 * kBM : kBM);
    p.n_tiles = (N + bn - 1) / bn;
    p.k_blocks = (K + kKE - 1) / kKE;
    p.units = p.m_tiles * p.n_tiles;
    const int waves = (p.units + slots - 1) / slots;
    p.cost = waves * (p.k_blocks * 2.0 * bn + 600.0);
    if (p.cost < best.cost) best = p;
  }
  return best;
}

template <class C>
cudaError_t launch_a16(const CUtensorMap& mx, const CUtensorMap& mw, const CUtensorMap& my,
                       const A16Params& p, int grid, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];  // per device; a repeated set is harmless
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(gemm_a16_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  if constexpr (C::PAIR) {
    // no more pairs than can be resident at once (a second, serial wave of a
    // persistent grid would only add a tail)
    static std::atomic<int> max_pairs[64];
    if (dev >= 0 && dev < 64 && max_pairs[dev].load(std::memory_order_acquire) == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(grid);
      cfg.blockDim = dim3(C::NUM_THREADS);
      cfg.dynamicSmemBytes = C::SMEM_BYTES;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_a16_kernel<C>, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1 << 20;  // unknown: keep the requested grid
      }
      max_pairs[dev].store(n, std::memory_order_release);
    }
    if (dev >= 0 && dev < 64) grid = std::min(grid, 2 * max_pairs[dev].load());
    return launch_pdl_cluster(gemm_a16_kernel<C>, dim3(grid), dim3(C::NUM_THREADS),
                              static_cast<size_t>(C::SMEM_BYTES), st, 2u, mx, mw, my, p);
  }
  return launch_pdl(gemm_a16_kernel<C>, dim3(grid), dim3(C::NUM_THREADS), C::SMEM_BYTES, st, mx,
                    mw, my, p);
}

template <bool W4, bool PAIR, bool PRE = false>
cudaError_t dispatch_a16(int bn, const CUtensorMap& mx, const CUtensorMap& mw,
                         const CUtensorMap& my, const A16Params& p, int grid, cudaStream_t st) {
  return bn == 128 ? launch_a16<A16Cfg<128, W4, PAIR, PRE>>(mx, mw, my, p, grid, st)
                   : launch_a16<A16Cfg<256, W4, PAIR, PRE>>(mx, mw, my, p, grid, st);
}

zq_status gemm_a16_entry(bool w4, const void* X, const void* Wq, const float* s_grp, int g,
                         const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                         zq_stream_t stream) {
  if (T < 0 || N < 8 || N % 8 != 0 || K < 16 || K % 16 != 0 || K > (1 << 20)) return ZQ_ERR_SHAPE;
  if (w4 && K % 32 != 0) return ZQ_ERR_SHAPE;
  if (g < 1 || g > N) return ZQ_ERR_SHAPE;
  if (T == 0) return ZQ_OK;
  if (!X || !Wq || !s_grp || !Y) return ZQ_ERR_NULL;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (acc_dbg && !aligned16(acc_dbg)))
    return ZQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // A handful of tokens: the CUDA-core matrix-vector path (the 128-row token
  // tile would leave the tensor cores nearly idle while the weights stream).
  const int forced_path = option(ZQ_OPT_GEMM_PATH);
  if (forced_path == 3 || (forced_path == 0 && T <= kGemvA16MaxTokens)) {
    if (T > kGemvA16MaxTokens) return ZQ_ERR_UNSUPPORTED;
    return launch_gemv_a16(w4 ? 4 : 8, X, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg,
                           option(ZQ_OPT_MAX_CTAS), st) == cudaSuccess
               ? ZQ_OK
               : ZQ_ERR_CUDA;
  }
  const int fbn = option(ZQ_OPT_GEMM_BN);
  if (fbn && fbn != 128 && fbn != 256) return ZQ_ERR_UNSUPPORTED;
  const int sms = num_sms();
  const int fpair = option(ZQ_OPT_CTA_PAIR);
  // Prefill-sized token counts: widen the codes once (an HBM-bound pass into
  // the library workspace), then a plain fp16 GEMM whose weight tiles arrive
  // by TMA; ZQ_OPT_GEMM_PATH = 4 forces it.
  const bool pre = forced_path == 4 || (forced_path == 0 && T >= kA16WidenMinTokens);
  A16Plan plan;
  if (pre) {
    // with nothing to widen in the tiles, CTA pairs halve the weight-tile
    // traffic per SM as in the INT8 GEMM: preferred for long rows
    const A16Plan single = plan_a16(T, N, K, sms, fbn, false);
    const A16Plan pr = plan_a16(T, N, K, sms, fbn, true);
    plan = fpair == 1 ? single
                      : (fpair == 2 || pr.cost * (K >= 2048 ? 0.82 : 1.10) < single.cost ? pr
                                                                                      : single);
  } else {
    // In-tile widening: CTA pairs halve the widening and the weight-tile
    // traffic per SM, but the cross-CTA handshake per stage costs more than
    // that saves (measured on B200: GPT-NeoX QKV at T = 4096 1.67 ms with
    // pairs, 1.39 ms without), so they run only when forced
    plan = plan_a16(T, N, K, sms, fbn, fpair == 2);
  }

  int* status = device_status_ptr();
  if (!status) return ZQ_ERR_CUDA;
  A16Params p{};
  p.s_grp = s_grp;
  p.bias = static_cast<const __half*>(bias);
  p.acc_dbg = acc_dbg;
  p.status = status;
  p.T = T;
  p.N = N;
  p.K = K;
  p.g = g;
  p.m_tiles = plan.m_tiles;
  p.n_tiles = plan.n_tiles;
  p.k_blocks = plan.k_blocks;
  p.num_units = plan.units;

  // fp16 activations [T][K] in the MMA's swizzled K-major layout; codes
  // int8 [N][K] or packed int4 [N][K/2] as plain rows; fp16 output [T][N]
  // in 32 x 32 blocks.
  const int code_row = w4 ? kKE / 2 : kKE;
  const uint64_t w_inner = w4 ? static_cast<uint64_t>(K) / 2 : static_cast<uint64_t>(K);
  const int w_box_rows = plan.pair ? plan.bn / 2 : plan.bn;
  const void* wsrc = Wq;
  if (pre) {
    void* wide = nullptr;
    const zq_status wrc = library_workspace(static_cast<size_t>(N) * K * 2, st, &wide);
    if (wrc != ZQ_OK) return wrc;
    const size_t n16 = static_cast<size_t>(N) * w_inner / 16;
    const int blocks = static_cast<int>(std::min<size_t>((n16 + 255) / 256, 8 * sms));
    const cudaError_t we =
        w4 ? launch_pdl(widen_a16_kernel<true>, dim3(std::max(blocks, 1)), dim3(256), 0, st,
                        static_cast<const uint4*>(Wq), static_cast<uint4*>(wide), n16)
           : launch_pdl(widen_a16_kernel<false>, dim3(std::max(blocks, 1)), dim3(256), 0, st,
                        static_cast<const uint4*>(Wq), static_cast<uint4*>(wide), n16);
    if (we != cudaSuccess) return ZQ_ERR_CUDA;
    wsrc = wide;
  }
  CUtensorMap mx, mw, my;
  if (!encode_tma_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, K, T, static_cast<uint64_t>(K) * 2,
                     kKE, kBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !(pre ? encode_tma_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wsrc, K, N,
                            static_cast<uint64_t>(K) * 2, kKE, w_box_rows,
                            CU_TENSOR_MAP_SWIZZLE_128B)
            : encode_tma_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, wsrc, w_inner, N, w_inner,
                            code_row, w_box_rows, CU_TENSOR_MAP_SWIZZLE_NONE)) ||
      !encode_tma_2d(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Y, N, T, static_cast<uint64_t>(N) * 2,
                     32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return ZQ_ERR_CUDA;

  int grid = std::min(plan.units, sms);
  const int cap = option(ZQ_OPT_MAX_CTAS);
  if (cap > 0) grid = std::min(grid, cap);
  if (plan.pair) {  // an even number of CTAs, one unit per pair at a time
    grid = 2 * std::min(plan.units, sms / 2);
    if (cap > 0) grid = std::min(grid, std::max(2, cap & ~1));
  }
  cudaError_t e;
  if (pre)
    e = plan.pair ? dispatch_a16<false, true, true>(plan.bn, mx, mw, my, p, grid, st)
                  : dispatch_a16<false, false, true>(plan.bn, mx, mw, my, p, grid, st);
  else if (plan.pair)
    e = w4 ? dispatch_a16<true, true>(plan.bn, mx, mw, my, p, grid, st)
           : dispatch_a16<false, true>(plan.bn, mx, mw, my, p, grid, st);
  else
    e = w4 ? dispatch_a16<true, false>(plan.bn, mx, mw, my, p, grid, st)
           : dispatch_a16<false, false>(plan.bn, mx, mw, my, p, grid, st);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

}  // namespace
}  // namespace zq

extern "C" zq_status zq_gemm_w8a16(const void* X, const int8_t* Wq, const float* s_grp, int g,
                                   const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                                   zq_stream_t stream) {
  return zq::gemm_a16_entry(false, X, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg, stream);
}

extern "C" zq_status zq_gemm_w4a16(const void* X, const uint8_t* Wq4, const float* s_grp, int g,
                                   const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                                   zq_stream_t stream) {
  return zq::gemm_a16_entry(true, X, Wq4, s_grp, g, bias, T, N, K, Y, acc_dbg, stream);
}
