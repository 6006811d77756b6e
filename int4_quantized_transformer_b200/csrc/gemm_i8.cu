// gemm_i8.cu -- W8A8 / W4A8 GEMM with the dequantization fused into the
// epilogue, on Blackwell tcgen05 tensor cores (ZeroQuant, arXiv 2206.01861,
// Sec. 3.4 "CUTLASS INT8 GEMM", "Dequantization fused into the GEMM
// epilogue", Fig. 2 right; INT4 FFN weights per "Which weights get INT4").
//
// One persistent, warp-specialised kernel serves both regimes the paper
// distinguishes ("Scheduling for different batch sizes"):
//
//  * token rows on the MMA M side (large T, tensor-bound): a 128 x BN tile
//    of Y per work unit, BN in {128, 192, 256} chosen to fill the 148 SMs;
//  * weight rows on the MMA M side (small T, weight-streaming, HBM-bound):
//    128 output features x all tokens (padded to BN in {16..256}) per unit,
//    with K split across SMs when there are fewer weight tiles than SMs.
//    Each split stores its exact int32 partial sums into a workspace; a
//    small second kernel, chained with programmatic dependent launch, adds
//    the splits (exact) and applies the dequant.  The mainloop never waits
//    on the reduction.
//
// Warp roles (one CTA per SM):
//   warp 0     TMA producer: activation and weight tiles, 128-byte K slices,
//              128B-swizzled, into a STAGES-deep mbarrier ring (with weight
//              rows on M, the last warp is a second producer: the two take
//              alternate K slices);
//   warp 1     TMEM allocator and MMA issuer: tcgen05.mma kind::i8, M=128,
//              N=BN, K=32, int32 accumulators in TMEM (two buffers, so the
//              epilogue of one unit overlaps the mainloop of the next);
//   warps 2-9  epilogue, two warps per TMEM lane quadrant, each taking half
//              of the columns: tcgen05.ld of the accumulator, then
//              y = fp16(((f32(acc)*s_tok[t]) * s_grp[group(o)]) + f32(bias[o]));
//              the scales and bias of a unit are loaded before its
//              accumulator is ready ("read the two groups of quantization
//              scales in advance");
//   warps 10-13 (W4A8 only) unpack: packed signed INT4 weights, staged by TMA,
//              are widened to int8 (as codes*16, two logic ops per eight
//              nibbles) and written into the MMA's 128B-swizzled K-major
//              layout in shared memory; the epilogue divides by 16 exactly.
//
// Every wait on an mbarrier is bounded (about a second), after which the
// kernel records the wait site in the device status word and every role
// leaves its loop; in-flight TMA copies and MMAs are drained before TMEM is
// released.  No barrier spans several warps inside the role loops, so a
// warp that gives up cannot strand another one.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "zq_internal.h"
#include "zq_ptx.cuh"

namespace zq {
namespace {

constexpr int BM = 128;       // MMA M: rows of a tile = TMEM lanes
constexpr int BK = 128;       // K bytes per pipeline stage (one swizzle row)
constexpr int UMMA_K = 32;    // K of one tcgen05.mma kind::i8
constexpr int kSmemBudget = 223 * 1024;
constexpr int NUM_EPI_WARPS_C = 8;
constexpr int kTmemUnpackWarps = 4;

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p *= 2;
  return p;
}

template <int BN_, bool WROWS_, bool W4_, bool PAIR_ = false>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr bool WROWS = WROWS_;  // weight rows on the MMA M side
  static constexpr bool W4 = W4_;
  // CTA pair (cta_group::2): a 256 x BN tile per pair; each CTA holds 128
  // token rows of A and BN/2 weight rows of B, and 128 rows of D in TMEM.
  static constexpr bool PAIR = PAIR_;
  static_assert(!PAIR || !WROWS, "CTA pairs serve the token-row tiling");
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;  // token rows per unit (token-row tiling)
  static constexpr int ACT_ROWS = WROWS ? BN : BM;
  static constexpr int W_ROWS = WROWS ? BM : (PAIR ? BN / 2 : BN);
  // Weight streaming with INT4 weights: the packed slices (with the small
  // activation tiles) get a deep ring of their own, so that many bytes are
  // in flight from HBM, while the unpacked weights use a shallow ring that
  // only the unpack warps and the MMA cycle through.
  // In this mode the deep ring holds, per stage, the packed weights and the
  // activation tiles (B); the shallow ring holds only unpacked weights (A).
  static constexpr bool DEEP = WROWS && W4;
  // K slices per pipeline stage.  INT4 weight streaming carries two (up to
  // BN = 128, where two deep slots of two slices still fit), so the
  // per-stage cost (waits, commits, the unpack handoff) is paid once per
  // 16 KB of packed weights instead of once per 8 KB.
  static constexpr int KPS = (DEEP && BN <= 128) ? 2 : 1;
  // TMEM columns per accumulator buffer: at least 32 so that the epilogue's
  // 32-column loads never leave the allocation.
  static constexpr int ACC_STRIDE = BN < 32 ? 32 : BN;
  static constexpr int BUF_COLS = ACC_STRIDE;  // TMEM columns per accumulator buffer
  // INT4 weight streaming up to BN = 128: the widened weights are written to
  // tensor memory and the MMA reads its A operand from there, so shared
  // memory carries only the packed codes and the activation tiles (it is
  // the bandwidth that bounds this path).  Their ring of slots sits in TMEM
  // after the two accumulator buffers, KPS * 32 columns per slot.
  static constexpr bool TMEM_A = DEEP && BN <= 128;
  static constexpr int A_COL0 = 2 * BUF_COLS;
  static constexpr int TMEM_A_SLOTS_RAW = (512 - 2 * BUF_COLS) / (32 * KPS);
  static constexpr int TMEM_A_SLOTS = TMEM_A_SLOTS_RAW > 4 ? 4 : TMEM_A_SLOTS_RAW;
  static constexpr int A_SLICE = BM * BK;                          // one K slice of A
  static constexpr int B_SLICE = (PAIR ? BN / 2 : BN) * BK;        // one K slice of B
  static constexpr int A_BYTES = TMEM_A ? 0 : A_SLICE * KPS;  // shared-memory A per stage
  static constexpr int B_BYTES = B_SLICE * KPS;
  static constexpr int P_BYTES = W4 ? W_ROWS * (BK / 2) * KPS : 0;  // packed row = KPS * 64 bytes
  // Weight streaming is bound by how fast TMA copies are issued: one issuing
  // thread per SM keeps well under the HBM bandwidth in flight, two do not.
  // The second producer warp is the last warp of the CTA; the producers take
  // alternate K slices, and the rings have an even number of slots so that
  // each slot is only ever filled by one of them.
  static constexpr int NUM_PROD_WARPS = WROWS ? 2 : 1;
  // columns handled by one epilogue warp (two warps share a lane quadrant)
  static constexpr int EPI_COLS = BN >= 64 ? BN / 2 : BN;
  // token-row tiling: per-warp staging of a 32 x 32 fp16 output block for
  // the TMA store (64-byte rows, 64-byte swizzle)
  static constexpr int STG_BYTES = WROWS ? 0 : 32 * 32 * 2;
  static constexpr int FREE_BYTES =
      kSmemBudget - NUM_EPI_WARPS_C * STG_BYTES - 8 * EPI_COLS * 8;
  static constexpr int STAGE_BYTES = DEEP ? A_BYTES : A_BYTES + B_BYTES + P_BYTES;
  static constexpr int STAGES_RAW =
      TMEM_A ? TMEM_A_SLOTS : (DEEP ? (KPS == 2 ? 2 : 4) : FREE_BYTES / STAGE_BYTES);
  static constexpr int STAGES_CAP = WROWS ? 12 : 8;
  static constexpr int STAGES_ANY = STAGES_RAW > STAGES_CAP ? STAGES_CAP : STAGES_RAW;
  // the producers fill the shallow ring only when there is no deep ring
  static constexpr int STAGES = (NUM_PROD_WARPS == 2 && !DEEP) ? STAGES_ANY & ~1 : STAGES_ANY;
  static constexpr int PSTAGES_RAW =
      DEEP ? (FREE_BYTES - STAGES * STAGE_BYTES) / (P_BYTES + B_BYTES) : STAGES;
  static constexpr int PSTAGES_ANY = PSTAGES_RAW > 16 ? 16 : PSTAGES_RAW;
  static constexpr int PSTAGES = DEEP ? PSTAGES_ANY & ~1 : PSTAGES_ANY;  // deep (packed) ring
  static constexpr int EPI_ARRIVALS = PAIR ? 2 * NUM_EPI_WARPS_C : NUM_EPI_WARPS_C;
  static constexpr int TMEM_COLS =
      pow2_at_least(2 * BUF_COLS + (TMEM_A ? STAGES * 32 * KPS : 0));
  static constexpr int NUM_EPI_WARPS = NUM_EPI_WARPS_C;
  // INT4 unpack warps: four (one per TMEM lane quadrant); with the TMEM
  // operand ring, kTmemUnpackWarps of them (eight: two per quadrant, each
  // widening one of the stage's two K slices)
  static constexpr int NUM_UNPACK_WARPS = W4 ? (TMEM_A ? kTmemUnpackWarps : 4) : 0;
  static constexpr int NUM_WARPS = 1 + NUM_PROD_WARPS + NUM_EPI_WARPS + NUM_UNPACK_WARPS;
  static constexpr int NUM_THREADS = 32 * NUM_WARPS;
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int P_RING = DEEP ? PSTAGES : STAGES;  // slots of the B and packed rings
  static constexpr int OFF_P = OFF_B + P_RING * B_BYTES;
  static constexpr int OFF_EPI = OFF_P + P_RING * P_BYTES;           // per-warp scale/bias
  static constexpr int EPI_BYTES = NUM_EPI_WARPS * EPI_COLS * 2 * 4;
  static constexpr int OFF_STG = ((OFF_EPI + EPI_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_BAR = OFF_STG + NUM_EPI_WARPS * STG_BYTES;
  static constexpr int NUM_BARS = 3 * STAGES + 2 * PSTAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(STAGES >= 2 && PSTAGES >= 2, "not enough shared memory for two stages");
  static_assert(NUM_PROD_WARPS == 1 || (DEEP ? PSTAGES % 2 == 0 : STAGES % 2 == 0),
                "two producers need rings with an even number of slots");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(!PAIR || (BN / 2) % 8 == 0, "B half-tile rows must fill 8-row swizzle atoms");
  static_assert(!W4 || (W_ROWS % (4 * NUM_UNPACK_WARPS) == 0 && (4 * NUM_UNPACK_WARPS) % 8 == 0),
                "unpack steps keep the row's swizzle phase");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(TMEM_COLS <= 512, "TMEM accumulators");
  static_assert(!TMEM_A || (KPS == 2 && STAGES >= 2 && P_BYTES == BM * 128 &&
                            A_COL0 + STAGES * 32 * KPS <= TMEM_COLS),
                "TMEM operand ring: packed rows of two K slices (128 bytes, 128B swizzle)");
  static_assert(EPI_COLS <= 128, "epilogue prefetch holds at most four columns per lane");
};

struct GemmParams {
  const float* s_tok;
  const float* s_grp;
  const __half* bias;
  __half* Y;
  int32_t* acc_dbg;
  int32_t* ws;     // split-K partial sums [splits][T][N]
  int* status;
  int T, N, K, g;
  int m_tiles, n_tiles, k_blocks, splits, num_units;
  int kps;  // K slices per pipeline stage (Cfg::KPS of the launched kernel)
  // Token-row tiling with a short last wave: the tiles from tail_start on
  // are split along K into tail_splits parts of tail_kb K slices each; their
  // exact int32 partial sums go to ws (tail tile j, part s at
  // ws + (j * tail_splits + s) * TILE_M * BN, row-major) and
  // tail_finalize_kernel adds them and dequantizes.  tail_start = the number
  // of tiles when there is no tail.
  int tail_start, tail_splits, tail_kb;
  // unit order: 0 = M tiles fastest (consecutive units, which run at the
  // same time, share their N-side operand tile), 1 = N tiles fastest
  int n_fastest;
  // INT4 weight streaming: map_act is a 3-D map that fetches the KPS
  // activation K slices of a stage in one box (K a multiple of KPS * 128)
  int act3d;
};

// A work unit: one output tile (m, n) and the K slices kb0, kb0 + kstep, ...
// below kb1.  With K split across SMs (weight-row tiling), split s of S
// takes the stages s, s + S, s + 2S, ... (stages of kps slices): at any
// moment the S CTAs of one weight tile read adjacent pieces of its rows,
// which the DRAM serves as longer contiguous runs than S separate ranges.
struct Unit {
  int m, n, kb0, kb1, kstep, split;
  int tail;  // index among the split tiles of the last wave, or -1
};

__device__ __forceinline__ Unit decode_unit(int u, const GemmParams& p) {
  Unit r;
  r.tail = -1;
  if (u >= p.tail_start) {  // a K part of a last-wave token-row tile
    const int j = u - p.tail_start;
    const int rest = p.tail_start + j / p.tail_splits;
    r.tail = j / p.tail_splits;
    r.split = j % p.tail_splits;
    r.m = rest % p.m_tiles;
    r.n = rest / p.m_tiles;
    r.kb0 = r.split * p.tail_kb;
    r.kb1 = min(p.k_blocks, r.kb0 + p.tail_kb);
    r.kstep = p.kps;
    return r;
  }
  const int split = u % p.splits;
  const int rest = u / p.splits;
  if (p.n_fastest) {
    r.n = rest % p.n_tiles;
    r.m = rest / p.n_tiles;
  } else {
    r.m = rest % p.m_tiles;
    r.n = rest / p.m_tiles;
  }
  r.split = split;
  r.kb0 = split * p.kps;
  r.kb1 = p.k_blocks;
  r.kstep = p.splits * p.kps;
  return r;
}

// group(o) = floor(o * g / N); a 32-bit division whenever o * g fits in 32
// bits (N * g < 2^32 covers every layer shape), else a 64-bit one.
__device__ __forceinline__ int group_of(int o, int N, int g) {
  const unsigned long long prod = static_cast<unsigned long long>(o) * static_cast<unsigned>(g);
  if (prod < (1ull << 32)) return static_cast<int>(static_cast<unsigned>(prod) / static_cast<unsigned>(N));
  return static_cast<int>(prod / static_cast<unsigned>(N));
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast, and
// __syncwarp orders the other lanes' later reads after lane 0's acquire.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status, int site) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status, site) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Widen one 32-bit word of packed INT4 codes (eight consecutive k: byte i
// holds k = i in its low nibble and k = 4 + i in its high nibble) to eight
// int8 values in k order.  Each nibble lands in the high half of its byte,
// so the bytes are the codes times 16 (exact two's complement, no carries
// between bytes); the epilogue divides the int32 accumulator by 16 exactly.
__device__ __forceinline__ void unpack8_x16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = (w << 4) & 0xF0F0F0F0u;  // k = 0..3
  hi = w & 0xF0F0F0F0u;         // k = 4..7
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __halves2half2(__float2half_rn(a), __float2half_rn(b));
  return *reinterpret_cast<uint32_t*>(&h);
}

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap map_act,
                   const __grid_constant__ CUtensorMap map_w,
                   const __grid_constant__ CUtensorMap map_y, const GemmParams p) {
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
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* ready_bar = bars + 2 * STAGES;  // W4: unpacked operand ready
  uint64_t* pfull_bar = bars + 3 * STAGES;      // [PSTAGES] packed INT4 slice landed (pairs, deep ring)
  uint64_t* pempty_bar = pfull_bar + C::PSTAGES;  // [PSTAGES] deep slot consumed by the MMA
  uint64_t* tfull_bar = pempty_bar + C::PSTAGES;  // [2]
  uint64_t* tempty_bar = tfull_bar + 2;     // [2]
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* flag_bcast = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  // CTA pairs: rank 0 (the leader) owns the full/tempty barriers and issues
  // the MMAs; units are numbered per pair.
  const uint32_t crank = C::PAIR ? cluster_ctarank() : 0u;
  const int unit0 = C::PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int ustep = C::PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&ready_bar[s], C::NUM_UNPACK_WARPS > 0
                                   ? (C::PAIR ? 2 : 1) * C::NUM_UNPACK_WARPS
                                   : 1);
    }
    for (int s = 0; s < C::PSTAGES; ++s) {
      mbar_init(&pfull_bar[s], 1);
      mbar_init(&pempty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], C::EPI_ARRIVALS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *flag_bcast = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_act);
    tma_prefetch_desc(&map_w);
    if (!C::WROWS) tma_prefetch_desc(&map_y);
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
  // Weight streaming: ask L2 for this CTA's first weight boxes before
  // waiting for the previous kernel of the stream (a fused LayerNorm +
  // quantization), so that the HBM stream starts while it runs.  Only L2 is
  // touched, which every kernel's writes reach coherently, so a weight
  // written by that kernel cannot be read stale.
  if (C::WROWS && threadIdx.x == 0 && static_cast<int>(unit0) < p.num_units) {
    const Unit t = decode_unit(unit0, p);
    for (int i = 0, kb = t.kb0; i < 12 && kb < t.kb1; ++i, kb += t.kstep)  // one box per stage
      tma_prefetch_l2_2d(&map_w, C::W4 ? kb * (BK / 2) : kb * BK, t.m * BM);
  }
  // Set-up above writes no global memory; everything below may read what
  // the previous kernel of the stream wrote, or overwrite what it reads.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0 || (C::NUM_PROD_WARPS == 2 && warp == C::NUM_WARPS - 1)) {
    // ------------------------------------------------------ TMA producer(s)
    // With two producers, producer `pid` issues the K slices whose running
    // index is congruent to pid modulo 2; both walk the same units and ring.
    constexpr int NP = C::NUM_PROD_WARPS;
    const int pid = warp == 0 ? 0 : 1;
    int seq = 0;
    if (C::DEEP && lane == 0) {
      // packed INT4 weight slice and activation tile of each K slice into
      // the deep ring
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_act = l2_policy_evict_last();
      constexpr uint32_t bytes = static_cast<uint32_t>(C::P_BYTES + C::B_BYTES);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[16];
      for (int s = 0; s < 16; ++s) fills[s] = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.num_units; u += ustep) {
        const Unit t = decode_unit(u, p);
        for (int kb = t.kb0; kb < t.kb1; kb += t.kstep) {
          if (NP > 1 && (seq++ % NP) != pid) {
            if (++stage == C::PSTAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          if (!mbar_wait(&pempty_bar[stage], phase ^ 1, abort_flag, p.status, 11)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&pfull_bar[stage], bytes);
          // KPS K slices: one packed box KPS*64 bytes wide, KPS activation
          // tiles (a slice past K reads the TMA's zero fill: it adds nothing)
          tma_load_2d(sP + stage * C::P_BYTES, &map_w, &pfull_bar[stage], kb * (BK / 2), t.m * BM,
                      pol_w);
          if (p.act3d) {
            tma_load_3d(sB + stage * C::B_BYTES, &map_act, &pfull_bar[stage], 0, t.n * BN, kb,
                        pol_act);
          } else {
#pragma unroll
            for (int h = 0; h < C::KPS; ++h)
              tma_load_2d(sB + stage * C::B_BYTES + h * C::B_SLICE, &map_act, &pfull_bar[stage],
                          (kb + h) * BK, t.n * BN, pol_act);
          }
          ++fills[stage];
          if (++stage == C::PSTAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      int no_abort = 0;
      for (int s = 0; s < C::PSTAGES; ++s)
        if (fills[s]) mbar_wait(&pfull_bar[s], (fills[s] - 1) & 1, &no_abort, p.status, 12);
    } else if (!C::DEEP && lane == 0) {
      const uint64_t pol_act = l2_policy_evict_last();
      // weights: streamed once when weight rows are the M side; in the
      // token-row tiling they are re-read by every token tile but can be far
      // larger than L2, so they get the first-to-go policy only in the former.
      const uint64_t pol_w = C::WROWS ? l2_policy_evict_first() : l2_policy_evict_normal();
      constexpr uint32_t act_bytes = C::ACT_ROWS * BK;
      constexpr uint32_t w_bytes = C::W4 ? C::P_BYTES : C::W_ROWS * BK;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[STAGES];
      for (int s = 0; s < STAGES; ++s) fills[s] = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.num_units; u += ustep) {
        const Unit t = decode_unit(u, p);
        const int act_row = C::WROWS ? t.n * BN : t.m * C::TILE_M + static_cast<int>(crank) * BM;
        const int w_row = C::WROWS ? t.m * BM : t.n * BN + static_cast<int>(crank) * C::W_ROWS;
        for (int kb = t.kb0; kb < t.kb1; kb += t.kstep) {
          if (NP > 1 && (seq++ % NP) != pid) {
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag, p.status, 1)) {
            ok = false;
            break;
          }
          if constexpr (C::PAIR) {
            // both CTAs' activation (and INT8 weight) bytes complete on the
            // leader's full barrier; packed INT4 weights on this CTA's own
            // pfull barrier, which its unpack warps wait on
            const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
            if (C::W4) {
              if (crank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * act_bytes);
              tma_load_2d_pair(sA + stage * C::A_BYTES, &map_act, fb, kb * BK, act_row, pol_act);
              mbar_arrive_expect_tx(&pfull_bar[stage], w_bytes);
              tma_load_2d(sP + stage * C::P_BYTES, &map_w, &pfull_bar[stage], kb * (BK / 2), w_row,
                          pol_w);
            } else {
              if (crank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * (act_bytes + w_bytes));
              tma_load_2d_pair(sA + stage * C::A_BYTES, &map_act, fb, kb * BK, act_row, pol_act);
              tma_load_2d_pair(sB + stage * C::B_BYTES, &map_w, fb, kb * BK, w_row, pol_w);
            }
            ++fills[stage];
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          mbar_arrive_expect_tx(&full_bar[stage], act_bytes + w_bytes);
          uint8_t* act_dst = C::WROWS ? sB + stage * C::B_BYTES : sA + stage * C::A_BYTES;
          tma_load_2d(act_dst, &map_act, &full_bar[stage], kb * BK, act_row, pol_act);
          if (C::W4) {
            tma_load_2d(sP + stage * C::P_BYTES, &map_w, &full_bar[stage], kb * (BK / 2), w_row,
                        pol_w);
          } else {
            uint8_t* w_dst = C::WROWS ? sA + stage * C::A_BYTES : sB + stage * C::B_BYTES;
            tma_load_2d(w_dst, &map_w, &full_bar[stage], kb * BK, w_row, pol_w);
          }
          ++fills[stage];
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Drain: every copy issued must land before the CTA exits (for a pair,
      // the leader's full barriers count both CTAs' copies; the follower
      // exits only after the final cluster barrier).
      int no_abort = 0;
      if (!C::PAIR || crank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (fills[s]) mbar_wait(&full_bar[s], (fills[s] - 1) & 1, &no_abort, p.status, 9);
      if (C::PAIR && C::W4)
        for (int s = 0; s < STAGES; ++s)
          if (fills[s]) mbar_wait(&pfull_bar[s], (fills[s] - 1) & 1, &no_abort, p.status, 10);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0 && (!C::PAIR || crank == 0)) {
      constexpr uint32_t idesc = make_idesc_i8(C::PAIR ? 2 * BM : BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int pst = 0;  // deep ring slot (activation tile)
      uint32_t pphase = 0;
      int buf = 0;
      uint32_t tphase = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.num_units; u += ustep) {
        const Unit t = decode_unit(u, p);
        if (!mbar_wait(&tempty_bar[buf], tphase ^ 1, abort_flag, p.status, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::BUF_COLS);
        for (int kb = t.kb0; kb < t.kb1; kb += t.kstep) {
          uint64_t* rb = C::W4 ? &ready_bar[stage] : &full_bar[stage];
          if (!mbar_wait(rb, phase, abort_flag, p.status, 3)) {
            ok = false;
            break;
          }
          // pairs with INT4 weights: the activations come on full, the
          // unpacked weights of both CTAs on ready.  Deep ring: the
          // activation tile sits in deep slot pst (landed with pfull).
          if (C::PAIR && C::W4 && !mbar_wait(&full_bar[stage], phase, abort_flag, p.status, 6)) {
            ok = false;
            break;
          }
          if (C::DEEP && !mbar_wait(&pfull_bar[pst], pphase, abort_flag, p.status, 7)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < C::KPS; ++h) {
            const uint64_t db = make_sw128_desc(
                smem_u32(sB + (C::DEEP ? pst : stage) * C::B_BYTES + h * C::B_SLICE));
            const bool first = kb == t.kb0 && h == 0;  // the unit's first K slice
            if constexpr (C::TMEM_A) {
              // A from TMEM: K = 32 bytes = 8 columns per MMA
              const uint32_t a_tm = tmem_base + static_cast<uint32_t>(
                                                    C::A_COL0 + (stage * C::KPS + h) * 32);
#pragma unroll
              for (int k = 0; k < BK / UMMA_K; ++k)
                mma_i8_ts(d_tmem, a_tm + static_cast<uint32_t>(8 * k),
                          db + static_cast<uint64_t>(2 * k), idesc, (!first || k > 0) ? 1u : 0u);
              continue;
            }
            const uint64_t da = make_sw128_desc(smem_u32(sA + stage * C::A_BYTES + h * C::A_SLICE));
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              // advance the start address by k*32 bytes (>>4 = 2k) inside the swizzle row
              if constexpr (C::PAIR)
                mma_i8_pair(d_tmem, da + static_cast<uint64_t>(2 * k),
                            db + static_cast<uint64_t>(2 * k), idesc, (!first || k > 0) ? 1u : 0u);
              else
                mma_i8(d_tmem, da + static_cast<uint64_t>(2 * k), db + static_cast<uint64_t>(2 * k),
                       idesc, (!first || k > 0) ? 1u : 0u);
            }
          }
          if constexpr (C::PAIR)
            mma_commit_pair_mc(&empty_bar[stage], 0x3);
          else
            mma_commit(&empty_bar[stage]);
          if constexpr (C::DEEP) {
            mma_commit(&pempty_bar[pst]);  // the deep slot (packed + activations) is free
            if (++pst == C::PSTAGES) {
              pst = 0;
              pphase ^= 1;
            }
          }
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
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      if constexpr (C::PAIR)
        mma_commit_pair_mc(drain_bar, 0x1);
      else
        mma_commit(drain_bar);
      int no_abort = 0;
      mbar_wait(drain_bar, 0, &no_abort, p.status, 8);
    }
  } else if (warp < 2 + C::NUM_EPI_WARPS) {
    // ------------------------------------------------------ epilogue
    // Two warps per TMEM lane quadrant (a warp may only read the 32 lanes of
    // quadrant warp%4); each takes half of the tile's columns.
    const int ew = warp - 2;          // epilogue warp index 0..7
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int half = ew >> 2;         // which half of the columns
    const int row_in_tile = quad * 32 + lane;
    constexpr bool kSplitCols = BN >= 64;
    const int cb = kSplitCols ? half * (BN / 2) : 0;                       // first column
    const int ce = kSplitCols ? cb + BN / 2 : (half == 0 ? BN : 0);        // one past the last
    // this warp's per-column scale and bias, indexed from its first column cb
    float* colv = sEpi + ew * (2 * C::EPI_COLS) - cb;
    float* colb = colv + C::EPI_COLS;
    uint8_t* stg = sStg + ew * C::STG_BYTES;
    int buf = 0;
    uint32_t tphase = 0;
    // A K split of the weight-row tiling stores raw partial sums and needs no
    // scales or bias.
    const bool split = C::WROWS && p.splits > 1;
    // The scales and bias of a unit are loaded into registers one unit ahead,
    // so their global-load latency overlaps the previous unit's epilogue
    // ("read the two groups of quantization scales in advance").  Lane l
    // holds columns cb + l + 32 i.
    constexpr int PCOLS = (C::EPI_COLS + 31) / 32;
    // bias stays in its fp16 form until used, so that nothing waits on the load
    float n_rs = 0.0f, n_cv[PCOLS];
    __half n_rb, n_cb[PCOLS];
    auto fetch = [&](int u) {
      n_rs = 0.0f;
      n_rb = __float2half_rn(0.0f);
#pragma unroll
      for (int i = 0; i < PCOLS; ++i) {
        n_cv[i] = 0.0f;
        n_cb[i] = __float2half_rn(0.0f);
      }
      if (u >= p.num_units || split) return;
      const Unit t = decode_unit(u, p);
      if (t.tail >= 0) return;  // a last-wave K part stores raw partial sums
      if (C::WROWS) {
        const int o = t.m * BM + row_in_tile;
        if (o < p.N) {
          n_rs = __ldg(p.s_grp + group_of(o, p.N, p.g));
          if (p.bias) n_rb = p.bias[o];
        }
#pragma unroll
        for (int i = 0; i < PCOLS; ++i) {
          const int c = cb + lane + 32 * i;
          const int tok = t.n * BN + c;
          if (c < ce && tok < p.T) n_cv[i] = __ldg(p.s_tok + tok);
        }
      } else {
        const int tok = t.m * C::TILE_M + static_cast<int>(crank) * BM + row_in_tile;
        if (tok < p.T) n_rs = __ldg(p.s_tok + tok);
#pragma unroll
        for (int i = 0; i < PCOLS; ++i) {
          const int c = cb + lane + 32 * i;
          const int o = t.n * BN + c;
          if (c < ce && o < p.N) {
            n_cv[i] = __ldg(p.s_grp + group_of(o, p.N, p.g));
            if (p.bias) n_cb[i] = p.bias[o];
          }
        }
      }
    };
    fetch(unit0);
    for (int u = unit0; u < p.num_units; u += ustep) {
      const Unit t = decode_unit(u, p);
      const float rscale = n_rs, rbias = __half2float(n_rb);
#pragma unroll
      for (int i = 0; i < PCOLS; ++i) {
        const int c = cb + lane + 32 * i;
        if (c < ce) {
          colv[c] = n_cv[i];
          colb[c] = __half2float(n_cb[i]);
        }
      }
      const int row_idx = C::WROWS ? t.m * BM + row_in_tile
                                   : t.m * C::TILE_M + static_cast<int>(crank) * BM + row_in_tile;
      __syncwarp();
      if (!wait_warp(&tfull_bar[buf], tphase, abort_flag, p.status, 4)) break;
      tc_fence_after();
      // the next unit's loads are in flight while this unit is processed
      fetch(u + ustep);
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(buf * C::BUF_COLS);

      auto process = [&](const uint32_t (&acc)[32], int c0) {
        if (C::WROWS) {
          // lane = output feature o, columns = tokens
          const int o = row_idx;
          if (o < p.N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tok = t.n * BN + c0 + j;
              if (c0 + j < BN && tok < p.T) {
                const int a = static_cast<int>(acc[j]);
                const size_t idx = static_cast<size_t>(tok) * p.N + o;
                if (split) {
                  p.ws[static_cast<size_t>(t.split) * p.T * p.N + idx] = a;
                } else {
                  float v = __fmul_rn(__int2float_rn(a), colv[c0 + j]);
                  v = __fadd_rn(__fmul_rn(v, rscale), rbias);
                  p.Y[idx] = __float2half_rn(v);
                  if (p.acc_dbg) p.acc_dbg[idx] = a;
                }
              }
            }
          }
        }
      };
      // token-row tiling, lane = token, columns = output features: dequantize
      // 32 accumulator columns into 16 packed fp16 pairs
      auto dequant_tok = [&](const uint32_t (&acc)[32], int c0, uint32_t (&h)[16]) {
        const int tok = row_idx;
        const int o0 = t.n * BN + c0;
        if (tok < p.T && o0 < p.N) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 sv = *reinterpret_cast<const float4*>(colv + c0 + j);
            const float4 bv = *reinterpret_cast<const float4*>(colb + c0 + j);
            float v0 = __fmul_rn(__int2float_rn(static_cast<int>(acc[j])), rscale);
            float v1 = __fmul_rn(__int2float_rn(static_cast<int>(acc[j + 1])), rscale);
            float v2 = __fmul_rn(__int2float_rn(static_cast<int>(acc[j + 2])), rscale);
            float v3 = __fmul_rn(__int2float_rn(static_cast<int>(acc[j + 3])), rscale);
            v0 = __fadd_rn(__fmul_rn(v0, sv.x), bv.x);
            v1 = __fadd_rn(__fmul_rn(v1, sv.y), bv.y);
            v2 = __fadd_rn(__fmul_rn(v2, sv.z), bv.z);
            v3 = __fadd_rn(__fmul_rn(v3, sv.w), bv.w);
            h[j / 2] = pack_half2(v0, v1);
            h[j / 2 + 1] = pack_half2(v2, v3);
          }
          int32_t* arow = p.acc_dbg ? p.acc_dbg + static_cast<size_t>(tok) * p.N + o0 : nullptr;
          if (arow) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (o0 + 8 * q < p.N) {  // N % 8 == 0: 8-column chunks are all in or all out
                reinterpret_cast<uint4*>(arow)[2 * q] =
                    make_uint4(acc[8 * q], acc[8 * q + 1], acc[8 * q + 2], acc[8 * q + 3]);
                reinterpret_cast<uint4*>(arow)[2 * q + 1] = make_uint4(
                    acc[8 * q + 4], acc[8 * q + 5], acc[8 * q + 6], acc[8 * q + 7]);
              }
            }
          }
        }
      };
      // The warp's 32 rows x 32 columns go out as one TMA tensor store (rows
      // past T / columns past N are clipped by the TMA unit): wait until the
      // previous store has read the staging buffer, write this lane's
      // 64-byte row in the 64B-swizzled layout, then issue.
      auto store_tok = [&](const uint32_t* h, int c0) {
        const int o0 = t.n * BN + c0;
        const int row0 = t.m * C::TILE_M + static_cast<int>(crank) * BM + quad * 32;
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

      if constexpr (C::WROWS) {
        // Two 32-column TMEM loads in flight before each wait.
#pragma unroll 1
        for (int c0 = cb; c0 < ce; c0 += 64) {
          uint32_t a0[32], a1[32];
          const bool two = c0 + 32 < ce;
          tmem_ld_32x32b_x32(t_row + c0, a0);
          if (two) tmem_ld_32x32b_x32(t_row + c0 + 32, a1);
          tmem_ld_wait();
          if (C::W4) {  // INT4 weights were widened as codes*16: exact division
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              a0[j] = static_cast<uint32_t>(static_cast<int>(a0[j]) >> 4);
              a1[j] = static_cast<uint32_t>(static_cast<int>(a1[j]) >> 4);
            }
          }
          process(a0, c0);
          if (two) process(a1, c0 + 32);
        }
      } else {
        // Token rows: dequantize and store 64 columns at a time, then release
        // the accumulator buffer.  (Dequantizing a warp's whole column range
        // into registers and releasing the buffer before the stores measured
        // slower: the stores then run back to back, each waiting for the
        // previous one to leave the staging buffer.)
#pragma unroll 1
        for (int c0 = cb; c0 < ce; c0 += 64) {
          uint32_t a0[32], a1[32];
          const bool two = c0 + 32 < ce;
          tmem_ld_32x32b_x32(t_row + c0, a0);
          if (two) tmem_ld_32x32b_x32(t_row + c0 + 32, a1);
          tmem_ld_wait();
          if (C::W4) {  // INT4 weights were widened as codes*16: exact division
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              a0[j] = static_cast<uint32_t>(static_cast<int>(a0[j]) >> 4);
              a1[j] = static_cast<uint32_t>(static_cast<int>(a1[j]) >> 4);
            }
          }
          if (!C::WROWS && t.tail >= 0) {
            // a K part of a last-wave tile: the exact int32 partial sums of
            // this lane's token row, 32 columns at a time (finalized by
            // tail_finalize_kernel)
            int32_t* prow = p.ws + (static_cast<size_t>(t.tail * p.tail_splits + t.split) * C::TILE_M +
                                    static_cast<int>(crank) * BM + row_in_tile) * BN + c0;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              reinterpret_cast<uint4*>(prow)[q] =
                  make_uint4(a0[4 * q], a0[4 * q + 1], a0[4 * q + 2], a0[4 * q + 3]);
            if (two) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                reinterpret_cast<uint4*>(prow + 32)[q] =
                    make_uint4(a1[4 * q], a1[4 * q + 1], a1[4 * q + 2], a1[4 * q + 3]);
            }
            continue;
          }
          uint32_t h[16];
          dequant_tok(a0, c0, h);
          store_tok(h, c0);
          if (two) {
            dequant_tok(a1, c0 + 32, h);
            store_tok(h, c0 + 32);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (C::PAIR)
            mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[buf]), 0));
          else
            mbar_arrive(&tempty_bar[buf]);
        }
      }
      if constexpr (C::WROWS) {
        // Release the accumulator buffer to the MMA warp.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty_bar[buf]);
      }
      if (++buf == 2) {
        buf = 0;
        tphase ^= 1;
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------ INT4 unpack (W4A8)
    if constexpr (C::W4) {
      const int ut = threadIdx.x - 32 * (2 + C::NUM_EPI_WARPS);  // 0 .. 32*NUM_UNPACK_WARPS-1
      constexpr int UROWS = 4 * C::NUM_UNPACK_WARPS;  // rows of one unpack step
      const int ur = ut >> 3, uj = ut & 7;
      constexpr int PROW = (BK / 2) * C::KPS;  // bytes of one packed row in a stage
      const int unp_src = ur * PROW + uj * 8;
      const int unp_dst = ur * BK + ((uj ^ (ur & 7)) << 4);
      int stage = 0;
      uint32_t phase = 0;
      int pst = 0;  // deep ring: packed slice
      uint32_t pphase = 0;
      bool ok = true;
      for (int u = unit0; ok && u < p.num_units; u += ustep) {
        const Unit t = decode_unit(u, p);
        for (int kb = t.kb0; kb < t.kb1; kb += t.kstep) {
          if constexpr (C::DEEP) {
            // the packed slice has landed, and the MMA has released the slot
            // of the shallow ring that the unpacked weights go to
            if (!wait_warp(&pfull_bar[pst], pphase, abort_flag, p.status, 13) ||
                !wait_warp(&empty_bar[stage], phase ^ 1, abort_flag, p.status, 14)) {
              ok = false;
              break;
            }
          } else if (!wait_warp(C::PAIR ? &pfull_bar[stage] : &full_bar[stage], phase, abort_flag,
                                p.status, 5)) {
            ok = false;
            break;
          }
          if constexpr (C::TMEM_A) {
            // Lane = weight row r of the tile, in this warp's TMEM lane
            // quadrant.  Its packed row (two K slices, 128 bytes, landed by
            // TMA in the 128B-swizzled layout: 16-byte chunk c of row r at
            // c ^ (r % 8)) is widened to codes*16 and written to the ring
            // slot's 2 x 32 TMEM columns (four k per column, in k order).
            const int r = (warp & 3) * 32 + lane;
            const uint8_t* prow = sP + pst * C::P_BYTES + r * PROW;
            const uint32_t a_tm = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                                  static_cast<uint32_t>(C::A_COL0 + stage * C::KPS * 32);
            // with two warps per quadrant, each widens one K slice of the stage
            constexpr int HPW = C::NUM_UNPACK_WARPS >= 4 * C::KPS ? 1 : C::KPS;  // slices per warp
            const int hb = HPW == 1 ? (ut / 128) : 0;
#pragma unroll
            for (int h = hb; h < hb + HPW; ++h) {
              uint32_t w[32];
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const uint4 v =
                    *reinterpret_cast<const uint4*>(prow + (((h * 4 + c) ^ (r & 7)) << 4));
                unpack8_x16(v.x, w[8 * c], w[8 * c + 1]);
                unpack8_x16(v.y, w[8 * c + 2], w[8 * c + 3]);
                unpack8_x16(v.z, w[8 * c + 4], w[8 * c + 5]);
                unpack8_x16(v.w, w[8 * c + 6], w[8 * c + 7]);
              }
              tmem_st_32x32b_x32(a_tm + static_cast<uint32_t>(h * 32), w);
            }
            tmem_st_wait();
            tc_fence_before();  // the stores are ordered before the MMA warp's reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready_bar[stage]);
            if (++pst == C::PSTAGES) {
              pst = 0;
              pphase ^= 1;
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          // Thread ut handles 16-byte output chunk j = ut % 8 of rows
          // r = ut / 8 + UROWS i: stepping a multiple of 8 rows keeps r % 8,
          // hence the swizzled chunk position, fixed, so the shared-memory
          // offsets are per-thread constants plus i * (UROWS rows).
#pragma unroll
          for (int h = 0; h < C::KPS; ++h) {
            const uint8_t* src = sP + (C::DEEP ? pst : stage) * C::P_BYTES + unp_src + h * (BK / 2);
            uint8_t* dst = (C::WROWS ? sA + stage * C::A_BYTES + h * C::A_SLICE
                                     : sB + stage * C::B_BYTES + h * C::B_SLICE) +
                           unp_dst;
#pragma unroll
            for (int i = 0; i < C::W_ROWS / UROWS; ++i) {
              const uint2 pk = *reinterpret_cast<const uint2*>(src + i * UROWS * PROW);
              uint4 o;
              unpack8_x16(pk.x, o.x, o.y);
              unpack8_x16(pk.y, o.z, o.w);
              *reinterpret_cast<uint4*>(dst + i * UROWS * BK) = o;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if constexpr (C::PAIR)
              mbar_arrive_cluster(mapa_shared(smem_u32(&ready_bar[stage]), 0));
            else
              mbar_arrive(&ready_bar[stage]);
          }
          if constexpr (C::DEEP) {
            if (++pst == C::PSTAGES) {
              pst = 0;
              pphase ^= 1;
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  }

  if (!C::WROWS && warp >= 2 && warp < 2 + C::NUM_EPI_WARPS && lane == 0) bulk_wait_group0();
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

// Split-K finalisation for the weight-row tiling: sum the int32 partial
// sums of the K splits (exact, in any order) and dequantize, four outputs
// per thread with four splits' loads in flight:
// y = fp16(((f32(acc) * s_tok[t]) * s_grp[group(o)]) + f32(bias[o])).
__global__ void __launch_bounds__(256)
    splitk_finalize_kernel(const int32_t* __restrict__ ws, int splits, const float* __restrict__ s_tok,
                           const float* __restrict__ s_grp, const __half* __restrict__ bias,
                           __half* __restrict__ Y, int32_t* __restrict__ acc_dbg, int T, int N,
                           int g) {
  // the partial sums are written by the GEMM kernel just before this one
  grid_dependency_wait();
  grid_launch_dependents();
  const size_t plane = static_cast<size_t>(T) * N;
  const size_t n4 = plane / 4;  // N % 8 == 0
  for (size_t v = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; v < n4;
       v += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t idx = v * 4;
    const int t = static_cast<int>(idx / N);
    const int o = static_cast<int>(idx - static_cast<size_t>(t) * N);
    const int4* src = reinterpret_cast<const int4*>(ws + idx);
    const size_t step = plane / 4;  // one split plane, in int4 units
    int4 acc = __ldcg(src);
    int sp = 1;
    for (; sp + 3 < splits; sp += 4) {
      const int4 a = __ldcg(src + sp * step), b = __ldcg(src + (sp + 1) * step);
      const int4 c = __ldcg(src + (sp + 2) * step), d = __ldcg(src + (sp + 3) * step);
      acc.x += (a.x + b.x) + (c.x + d.x);
      acc.y += (a.y + b.y) + (c.y + d.y);
      acc.z += (a.z + b.z) + (c.z + d.z);
      acc.w += (a.w + b.w) + (c.w + d.w);
    }
    for (; sp < splits; ++sp) {
      const int4 a = __ldcg(src + sp * step);
      acc.x += a.x; acc.y += a.y; acc.z += a.z; acc.w += a.w;
    }
    const int av[4] = {acc.x, acc.y, acc.z, acc.w};
    const float st = __ldg(s_tok + t);
    uint32_t h[2];
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      float v0 = __fmul_rn(__int2float_rn(av[j]), st);
      float v1 = __fmul_rn(__int2float_rn(av[j + 1]), st);
      v0 = __fadd_rn(__fmul_rn(v0, __ldg(s_grp + group_of(o + j, N, g))),
                     bias ? __half2float(bias[o + j]) : 0.0f);
      v1 = __fadd_rn(__fmul_rn(v1, __ldg(s_grp + group_of(o + j + 1, N, g))),
                     bias ? __half2float(bias[o + j + 1]) : 0.0f);
      h[j / 2] = pack_half2(v0, v1);
    }
    *reinterpret_cast<uint2*>(Y + idx) = make_uint2(h[0], h[1]);
    if (acc_dbg) *reinterpret_cast<int4*>(acc_dbg + idx) = acc;
  }
}

// The last-wave tiles of the token-row tiling, split along K: add each
// output's int32 partial sums (exact) and dequantize, eight outputs per
// thread, y = fp16(((f32(acc) * s_tok[t]) * s_grp[group(o)]) + f32(bias[o])).
// Partials of tail tile j, part s: ws + (j * splits + s) * tile_m * bn,
// row-major [tile_m][bn].
__global__ void __launch_bounds__(256)
    tail_finalize_kernel(const int32_t* __restrict__ ws, int ntail, int splits, int tail_start,
                         int m_tiles, int tile_m, int bn, const float* __restrict__ s_tok,
                         const float* __restrict__ s_grp, const __half* __restrict__ bias,
                         __half* __restrict__ Y, int32_t* __restrict__ acc_dbg, int T, int N,
                         int g) {
  // the partial sums are written by the GEMM kernel just before this one
  grid_dependency_wait();
  grid_launch_dependents();
  const size_t tile_elems = static_cast<size_t>(tile_m) * bn;
  const size_t n8 = static_cast<size_t>(ntail) * tile_elems / 8;  // bn % 8 == 0
  for (size_t v = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; v < n8;
       v += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t e = v * 8;
    const int j = static_cast<int>(e / tile_elems);
    const int within = static_cast<int>(e - static_cast<size_t>(j) * tile_elems);
    const int lrow = within / bn, lcol = within - lrow * bn;
    const int tile = tail_start + j;
    const int t = (tile % m_tiles) * tile_m + lrow;
    const int o = (tile / m_tiles) * bn + lcol;
    if (t >= T || o >= N) continue;  // N % 8 == 0: eight columns are all in or all out
    const int32_t* src = ws + static_cast<size_t>(j) * splits * tile_elems + within;
    int4 lo = __ldcg(reinterpret_cast<const int4*>(src));
    int4 hi = __ldcg(reinterpret_cast<const int4*>(src) + 1);
    for (int sp = 1; sp < splits; ++sp) {
      const int4* q = reinterpret_cast<const int4*>(src + sp * tile_elems);
      const int4 a = __ldcg(q), b = __ldcg(q + 1);
      lo.x += a.x; lo.y += a.y; lo.z += a.z; lo.w += a.w;
      hi.x += b.x; hi.y += b.y; hi.z += b.z; hi.w += b.w;
    }
    const int acc[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const float st = __ldg(s_tok + t);
    uint32_t h[4];
#pragma unroll
    for (int q = 0; q < 8; q += 2) {
      float v0 = __fmul_rn(__int2float_rn(acc[q]), st);
      float v1 = __fmul_rn(__int2float_rn(acc[q + 1]), st);
      v0 = __fadd_rn(__fmul_rn(v0, __ldg(s_grp + group_of(o + q, N, g))),
                     bias ? __half2float(bias[o + q]) : 0.0f);
      v1 = __fadd_rn(__fmul_rn(v1, __ldg(s_grp + group_of(o + q + 1, N, g))),
                     bias ? __half2float(bias[o + q + 1]) : 0.0f);
      h[q / 2] = pack_half2(v0, v1);
    }
    const size_t idx = static_cast<size_t>(t) * N + o;
    *reinterpret_cast<uint4*>(Y + idx) = make_uint4(h[0], h[1], h[2], h[3]);
    if (acc_dbg) {
      reinterpret_cast<int4*>(acc_dbg + idx)[0] = lo;
      reinterpret_cast<int4*>(acc_dbg + idx)[1] = hi;
    }
  }
}

// INT4 weights for prefill-sized token counts: the packed codes are widened
// once per call to int8 codes in a workspace, [N][K] in k order, and the
// INT8 GEMM reads them from there.  Each weight tile is then widened once
// instead of once per token tile, and the GEMM's shared memory carries only
// the TMA copies and the MMA operand reads (the widening inside the tiles,
// through shared memory or into tensor memory, competes with both).  The
// pass is HBM-bound: N*K/2 bytes read and N*K written.
//
// Of each 32-bit word of packed codes (eight consecutive k), byte i holds
// k = i in its low nibble and k = 4 + i in its high nibble; a nibble n is the
// two's-complement code n - 16 * (n >= 8), i.e. the byte n | 0xF0 when bit 3
// is set (the mask times 0x1E sets the four high bits of exactly those
// bytes, with no carry between bytes).
__device__ __forceinline__ uint32_t sext_nibbles(uint32_t n) {
  return n | ((n & 0x08080808u) * 0x1Eu);
}

constexpr int kWidenUnroll = 4;  // 16-byte loads in flight per thread

__device__ __forceinline__ void widen_store(uint4 w, uint4* dst) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t out[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    out[2 * m] = sext_nibbles(in[m] & 0x0F0F0F0Fu);             // k = 8m .. 8m + 3
    out[2 * m + 1] = sext_nibbles((in[m] >> 4) & 0x0F0F0F0Fu);  // k = 8m + 4 .. 8m + 7
  }
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
}

__global__ void __launch_bounds__(256)
    widen_w4_kernel(const uint4* __restrict__ packed, uint4* __restrict__ wide, size_t n16) {
  // the packed codes may be written by the previous kernel of the stream
  grid_dependency_wait();
  grid_launch_dependents();
  // each thread keeps kWidenUnroll loads in flight (a 16-byte chunk = 32
  // codes: k = 32i .. 32i + 31 of one row), so the pass runs at the HBM rate
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  for (; i + (kWidenUnroll - 1) * stride < n16; i += kWidenUnroll * stride) {
    uint4 w[kWidenUnroll];
#pragma unroll
    for (int u = 0; u < kWidenUnroll; ++u) w[u] = __ldcs(packed + i + u * stride);
#pragma unroll
    for (int u = 0; u < kWidenUnroll; ++u) widen_store(w[u], wide + 2 * (i + u * stride));
  }
  for (; i < n16; i += stride) widen_store(__ldcs(packed + i), wide + 2 * i);
}

// ------------------------------------------------------------------ host

// The library workspace of one device.  Growing it allocates a new buffer
// and retires the old one without freeing it: kernels recorded into a CUDA
// graph before the growth keep their pointers into the old buffer, and the
// graph stays valid.  Retired buffers are released when the process exits.
// Each growth takes at least a quarter more than the last size, so the
// retired buffers together hold less than four times the final size.
struct Workspace {
  int32_t* ws = nullptr;
  size_t ws_elems = 0;
  std::vector<void*> retired;
};
std::mutex g_ws_mu;
Workspace g_ws[64];

constexpr size_t kWorkspaceGranule = size_t(1) << 19;  // int32 elements (2 MiB)

// A workspace of at least `elems` int32 elements on the current device.
// `check_capture`: refuse (ZQ_ERR_UNSUPPORTED) to grow while `st` is being
// captured into a CUDA graph, since an allocation would end the capture.
zq_status ensure_workspace(size_t elems, bool check_capture, cudaStream_t st, int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return ZQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  Workspace& w = g_ws[dev];
  if (w.ws_elems < elems) {
    if (check_capture) {
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
        return ZQ_ERR_UNSUPPORTED;
    }
    size_t want = std::max(elems, w.ws_elems + w.ws_elems / 4);
    want = (want + kWorkspaceGranule - 1) / kWorkspaceGranule * kWorkspaceGranule;
    int32_t* p = nullptr;
    if (cudaMalloc(&p, want * sizeof(int32_t)) != cudaSuccess) {
      cudaGetLastError();  // the failed allocation is reported, not left sticky
      return ZQ_ERR_CUDA;
    }
    if (w.ws) w.retired.push_back(w.ws);
    w.ws = p;
    w.ws_elems = want;
  }
  *out = w.ws;
  return ZQ_OK;
}

}  // namespace

zq_status library_workspace(size_t bytes, cudaStream_t st, void** out) {
  int32_t* p = nullptr;
  const zq_status rc = ensure_workspace((bytes + 3) / 4, true, st, &p);
  if (rc == ZQ_OK) *out = p;
  return rc;
}

namespace {

// The split-K finalisation, launched right after the GEMM kernel on the same
// stream (programmatic dependent launch: it is scheduled early and waits in
// the kernel for the GEMM's partial sums).
cudaError_t launch_finalize(const GemmParams& gp, cudaStream_t st) {
  const size_t n4 = static_cast<size_t>(gp.T) * gp.N / 4;
  const int blocks = static_cast<int>(std::min<size_t>((n4 + 255) / 256, 8 * num_sms()));
  return launch_pdl(splitk_finalize_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, st,
                    static_cast<const int32_t*>(gp.ws), gp.splits, gp.s_tok, gp.s_grp, gp.bias,
                    gp.Y, gp.acc_dbg, gp.T, gp.N, gp.g);
}

struct Plan {
  bool wrows;
  bool pair;
  int bn;
  int m_tiles, n_tiles, k_blocks, splits, kb_per_split, units;
  int kps = 1;  // K slices per pipeline stage (weight rows with INT4 weights: 2)
  // token rows: tiles from tail_start on (the last, short wave) are split
  // along K into tail_splits parts of tail_kb slices (tail_start = the tile
  // count when there is no such split)
  int tail_start = 0, tail_splits = 1, tail_kb = 0;
  double cost;
};

int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// Largest token count the automatic choice sends to the matrix-vector path.
int gemv_max_tokens(bool w4) { return w4 ? kGemvMaxTokens : 2; }

// The automatic choice of weight rows on the MMA M side (above the
// matrix-vector range).  INT8 weights: up to 256 tokens (weight streaming).
// INT4 weights: up to 128 tokens, where the widened weights live in tensor
// memory next to the accumulators; from 512 tokens the widening pass and
// the INT8 GEMM take over (kWidenMinTokens), and in between the token-row
// tiles widen the weights through shared memory.
bool use_weight_rows(int T, int K, bool w4) {
  (void)K;
  if (!w4) return T <= 256;
  return T <= 128;
}

// fp16 output [T][N]: 32 x 32 boxes written by the epilogue warps
bool encode_y_map(CUtensorMap* my, void* Y, int T, int N) {
  return encode_tma_2d(my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Y, N, T, static_cast<uint64_t>(N) * 2,
                       32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// Wave-aware cost in MMA cycles: ceil(units/SMs) * k-blocks per unit * 2*BN
// (a 128 x BN x 128 int8 block takes about 2*BN cycles), plus a fixed
// charge per extra wave and per split-K reduction.
// K is split in whole stages of kps K slices: two for INT4 weights up to
// BN = 128 (Cfg::KPS), else one.
Plan plan_wrows(int T, int N, int K, int sms, int forced_split, bool w4) {
  Plan p{};
  p.wrows = true;
  p.pair = false;
  // INT4 weights: at most 128 tokens per tile, so that the widened weights
  // can live in tensor memory next to the two accumulator buffers
  const int bn_cap = w4 ? 128 : 256;
  int bn = 16;
  while (bn < T && bn < bn_cap) bn *= 2;
  p.bn = bn;
  const int kps = (w4 && bn <= 128) ? 2 : 1;
  p.kps = kps;
  p.m_tiles = ceil_div(N, BM);
  p.n_tiles = ceil_div(T, bn);
  p.k_blocks = ceil_div(K, BK);
  const int tiles = p.m_tiles * p.n_tiles;
  const int k_stages = ceil_div(p.k_blocks, kps);
  double best = 1e30;
  int best_s = 1;
  const int max_s = forced_split > 0 ? std::min(forced_split, k_stages) : std::min(k_stages, 32);
  const int min_s = forced_split > 0 ? max_s : 1;
  for (int s = min_s; s <= max_s; ++s) {
    const int sps = ceil_div(k_stages, s);  // stages per split
    const int s_eff = ceil_div(k_stages, sps);
    const int units = tiles * s_eff;
    const int waves = ceil_div(units, sms);
    double cost;
    if (w4) {
      // the unit time is set by its widening pipeline: count stages
      cost = waves * (sps * kps + 2.0) + (s_eff > 1 ? 1.0 : 0.0);
    } else {
      // INT8 weights, in microseconds (fitted to B200 kernel timings after an
      // L2 flush, T = 8 to 64): the weights stream at the lower of 5.5 TB/s
      // over the GPU and 55 GB/s into one CTA (the operand bytes of its
      // stages); a K split costs 3 us + 0.1 us per token column of the tile
      // (the partial sums' stores and the finalize kernel), and each further
      // unit a persistent CTA takes on about 0.9 us
      const double w_stage = static_cast<double>(BM) * BK;
      const double cta_bytes = waves * sps * (w_stage + static_cast<double>(bn) * BK);
      const double all_bytes = static_cast<double>(tiles) * k_stages * w_stage;
      cost = std::max(all_bytes / 5.5e6, cta_bytes / 5.5e4) +
             (s_eff > 1 ? 3.0 + 0.1 * bn : 0.0) + 0.9 * (waves - 1);
    }
    if (cost < best - 1e-9) {
      best = cost;
      best_s = s_eff;
    }
  }
  p.kb_per_split = kps * ceil_div(k_stages, best_s);
  p.splits = ceil_div(p.k_blocks, p.kb_per_split);
  p.units = tiles * p.splits;
  p.cost = best * 2.0 * 256;  // comparable scale with the token-row plan
  return p;
}

// Token-row tiling: 128 x BN tiles per CTA, or 256 x BN tiles per CTA pair
// (each CTA of the pair does the same MMA work as a single-CTA tile, so a
// unit costs the same; there are half as many "slots").
Plan plan_trows(int T, int N, int K, int sms, int forced_bn, bool pair, bool allow_tail,
                int forced_tail) {
  Plan best{};
  best.cost = 1e30;
  const int cands[3] = {256, 192, 128};
  const int slots = pair ? sms / 2 : sms;
  for (int bn : cands) {
    if (forced_bn && bn != forced_bn) continue;
    Plan p{};
    p.wrows = false;
    p.pair = pair;
    p.bn = bn;
    p.m_tiles = ceil_div(T, pair ? 2 * BM : BM);
    p.n_tiles = ceil_div(N, bn);
    p.k_blocks = ceil_div(K, BK);
    p.splits = 1;
    p.kb_per_split = p.k_blocks;
    p.units = p.m_tiles * p.n_tiles;
    p.tail_start = p.units;
    const int waves = ceil_div(p.units, slots);
    p.cost = waves * (p.k_blocks * 2.0 * bn + 600.0);
    // A last wave less than half full: split its tiles along K over the idle
    // slots (parts of at least four K slices), so that wave takes a fraction
    // of a tile's time; a finalize kernel adds the parts.  Only 256-wide
    // tiles: narrower ones cost more per MAC than the cost model counts
    // (measured on B200: 256 x 192 and 256 x 128 CTA-pair tiles 1.1x and
    // 1.5x the time per MAC of 256 x 256 ones), and the finalize launch is
    // charged about 2 us.
    // Measured on GPT-NeoX at T = 4096: FFN2 (K = 24576) 449 -> 401 us with the
    // split, attention-out (K = 6144) unchanged (its finalize cost what the
    // shorter wave saved), so it is automatic for long rows only;
    // ZQ_OPT_SPLIT_K > 1 forces it (that many parts) whenever the last wave
    // is partial.
    const int full = p.units / slots, rem = p.units % slots;
    const bool forced = forced_tail > 1 && rem > 0 && full >= 1;
    if (allow_tail && (forced || (bn == 256 && p.k_blocks >= 96 && full >= 1 && rem > 0 &&
                                  2 * rem <= slots))) {
      const int want = forced ? std::min(forced_tail, p.k_blocks)
                              : std::min(std::min(slots / rem, p.k_blocks / 4), 8);
      if (want >= 2) {
        p.tail_kb = ceil_div(p.k_blocks, want);
        p.tail_splits = ceil_div(p.k_blocks, p.tail_kb);
        p.tail_start = full * slots;
        p.units = p.tail_start + rem * p.tail_splits;
        p.cost = full * (p.k_blocks * 2.0 * bn + 600.0) + (p.tail_kb * 2.0 * bn + 600.0) + 4000.0;
      }
    }
    if (p.cost < best.cost) best = p;
  }
  return best;
}

template <class C>
cudaError_t launch_cfg(const CUtensorMap& ma, const CUtensorMap& mw, const CUtensorMap& my,
                       const GemmParams& gp, int grid, cudaStream_t st) {
  // grid: CTAs requested; clamped below for CTA pairs
  // per device and kernel variant; several host threads may race here, and
  // setting the attribute twice is harmless
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_i8_kernel<C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  if constexpr (C::PAIR) {
    // A persistent grid of pairs larger than the number of pairs that can be
    // resident at once would leave a second, serial wave: clamp to it.
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
      if (cudaOccupancyMaxActiveClusters(&n, gemm_i8_kernel<C>, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1 << 20;  // unknown: keep the requested grid
      }
      max_pairs[dev].store(n, std::memory_order_release);
    }
    if (dev >= 0 && dev < 64) grid = std::min(grid, 2 * max_pairs[dev].load());
  }
  cudaError_t e =
      C::PAIR ? launch_pdl_cluster(gemm_i8_kernel<C>, dim3(grid), dim3(C::NUM_THREADS),
                                   static_cast<size_t>(C::SMEM_BYTES), st, 2u, ma, mw, my, gp)
              : launch_pdl(gemm_i8_kernel<C>, dim3(grid), dim3(C::NUM_THREADS),
                           static_cast<size_t>(C::SMEM_BYTES), st, ma, mw, my, gp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool W4>
cudaError_t dispatch_pair(int bn, const CUtensorMap& ma, const CUtensorMap& mw,
                          const CUtensorMap& my, const GemmParams& gp, int grid, cudaStream_t st) {
  switch (bn) {
    case 128: return launch_cfg<Cfg<128, false, W4, true>>(ma, mw, my, gp, grid, st);
    case 192: return launch_cfg<Cfg<192, false, W4, true>>(ma, mw, my, gp, grid, st);
    default: return launch_cfg<Cfg<256, false, W4, true>>(ma, mw, my, gp, grid, st);
  }
}

template <bool WROWS, bool W4>
cudaError_t dispatch_bn(int bn, const CUtensorMap& ma, const CUtensorMap& mw,
                        const CUtensorMap& my, const GemmParams& gp, int grid, cudaStream_t st) {
  if constexpr (WROWS) {
    switch (bn) {
      case 16: return launch_cfg<Cfg<16, true, W4>>(ma, mw, my, gp, grid, st);
      case 32: return launch_cfg<Cfg<32, true, W4>>(ma, mw, my, gp, grid, st);
      case 64: return launch_cfg<Cfg<64, true, W4>>(ma, mw, my, gp, grid, st);
      case 128: return launch_cfg<Cfg<128, true, W4>>(ma, mw, my, gp, grid, st);
      default: return launch_cfg<Cfg<256, true, W4>>(ma, mw, my, gp, grid, st);
    }
  } else {
    switch (bn) {
      case 128: return launch_cfg<Cfg<128, false, W4>>(ma, mw, my, gp, grid, st);
      case 192: return launch_cfg<Cfg<192, false, W4>>(ma, mw, my, gp, grid, st);
      default: return launch_cfg<Cfg<256, false, W4>>(ma, mw, my, gp, grid, st);
    }
  }
}

// The checks shared by every GEMM entry point (synchronous, before any
// launch).
zq_status check_gemm_args(bool w4, const int8_t* Xq, const float* s_tok, const void* Wq,
                          const float* s_grp, int g, const void* bias, int T, int N, int K,
                          const void* Y, const int32_t* acc_dbg) {
  if (T < 0 || N < 8 || N % 8 != 0 || K < 16 || K % 16 != 0 || K > 133136) return ZQ_ERR_SHAPE;
  if (w4 && (K % 32 != 0 || K > 132096)) return ZQ_ERR_SHAPE;
  if (g < 1 || g > N) return ZQ_ERR_SHAPE;
  if (T == 0) return ZQ_OK;
  if (!Xq || !s_tok || !Wq || !s_grp || !Y) return ZQ_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (acc_dbg && !aligned16(acc_dbg)))
    return ZQ_ERR_ALIGN;
  return ZQ_OK;
}

// The kernel a call runs: the CUDA-core matrix-vector path, or a tensor-core
// plan.  forced_split > 0 fixes the number of K splits of a weight-row plan.
struct Choice {
  bool gemv = false;
  bool widen = false;  // INT4 weights widened into the workspace, then the INT8 plan
  Plan plan{};
};

// INT4 weights at prefill-sized token counts take the widening pass and the
// INT8 GEMM (widen_w4_kernel).  Measured on B200 (GPT-NeoX FFN1/FFN2): at 512
// tokens 107/117 us against 121/135 us for the token-row tiles that widen
// through shared memory; at 256 tokens the tiles are ahead (79 against
// 123 us), the pass then being a third of the time.
constexpr int kWidenMinTokens = 512;

zq_status choose(bool w4, int T, int N, int K, int forced_split, Choice* out,
                 bool allow_tail = true) {
  const int sms = num_sms();
  // A handful of tokens: the CUDA-core matrix-vector path (measured faster
  // than the tensor-core tilings up to T = 4 with INT4 weights and up to
  // T = 2 with INT8 ones).  Otherwise weight rows on the MMA M side for small
  // token counts (weight streaming), token rows beyond; tests and benchmarks
  // may force any of them.
  int forced_path = option(ZQ_OPT_GEMM_PATH);
  out->widen = false;
  if (forced_path == 4 && !w4) return ZQ_ERR_UNSUPPORTED;
  if (w4 && (forced_path == 4 || (forced_path == 0 && T >= kWidenMinTokens))) {
    // the INT8 GEMM on the widened codes, planned as for INT8 weights
    out->widen = true;
    w4 = false;
    forced_path = 0;
  }
  if (forced_path == 3 || (forced_path == 0 && T <= gemv_max_tokens(w4))) {
    if (T > kGemvMaxTokens) return ZQ_ERR_UNSUPPORTED;
    out->gemv = true;
    return ZQ_OK;
  }
  out->gemv = false;
  if (forced_path == 2 || (forced_path == 0 && use_weight_rows(T, K, w4))) {
    out->plan = plan_wrows(T, N, K, sms, forced_split, w4);
    return ZQ_OK;
  }
  const int fbn = option(ZQ_OPT_GEMM_BN);
  if (fbn && fbn != 128 && fbn != 192 && fbn != 256) return ZQ_ERR_UNSUPPORTED;
  // CTA pairs need less operand traffic per SM (32 KB instead of 48 KB per
  // 128-deep K slice) but pay a cross-CTA handshake per stage and per
  // tile.  Measured on B200 over the layer shapes: pairs of 256 x 256
  // tiles run ~18% faster per tile when K >= 2048 and ~10% slower at small
  // K, so the two wave-aware plans are compared with those factors.
  const int fpair = option(ZQ_OPT_CTA_PAIR);
  const Plan single = plan_trows(T, N, K, sms, fbn, false, allow_tail, forced_split);
  if (fpair == 1) {
    out->plan = single;
    return ZQ_OK;
  }
  const Plan pr = plan_trows(T, N, K, sms, fbn ? fbn : 256, true, allow_tail, forced_split);
  // INT4: the unpack stage, not the operand feed, bounds the mainloop;
  // pairs measured slower there, so they are used only when forced.
  const double f = w4 ? 1e9 : (K >= 2048 ? 0.82 : 1.10);
  out->plan = (fpair == 2 || pr.cost * f < single.cost) ? pr : single;
  return ZQ_OK;
}

// Last-wave tiles a token-row plan splits along K.
int tail_tiles(const Plan& plan) {
  return plan.wrows ? 0 : (plan.units - plan.tail_start) / plan.tail_splits;
}

// Partial sums a plan stores (int32 elements): a weight-row plan with K
// splits, or the K parts of a token-row plan's last-wave tiles.
size_t split_partials(const Plan& plan, int T, int N) {
  if (plan.wrows) return plan.splits > 1 ? static_cast<size_t>(plan.splits) * T * N : 0;
  return static_cast<size_t>(tail_tiles(plan)) * plan.tail_splits * (plan.pair ? 2 * BM : BM) *
         plan.bn;
}

// The finalisation of the last-wave tiles, chained after the GEMM kernel.
cudaError_t launch_tail_finalize(const GemmParams& gp, const Plan& plan, cudaStream_t st) {
  const int ntail = tail_tiles(plan);
  const int tile_m = plan.pair ? 2 * BM : BM;
  const size_t n8 = static_cast<size_t>(ntail) * tile_m * plan.bn / 8;
  const int blocks = static_cast<int>(std::min<size_t>((n8 + 255) / 256, 4 * 148));
  return launch_pdl(tail_finalize_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, st,
                    static_cast<const int32_t*>(gp.ws), ntail, plan.tail_splits, plan.tail_start,
                    gp.m_tiles, tile_m, plan.bn, gp.s_tok, gp.s_grp, gp.bias, gp.Y, gp.acc_dbg, gp.T,
                    gp.N, gp.g);
}

// Launches a chosen plan; `ws` receives the split-K partial sums (at least
// split_partials() elements) when the plan splits K.
zq_status launch_choice(bool w4, const Choice& ch, const int8_t* Xq, const float* s_tok,
                        const void* Wq, const float* s_grp, int g, const void* bias, int T, int N,
                        int K, void* Y, int32_t* acc_dbg, int32_t* ws, cudaStream_t st) {
  if (ch.gemv)
    return launch_gemv_i8(w4 ? 4 : 8, Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg,
                          option(ZQ_OPT_MAX_CTAS), st) == cudaSuccess
               ? ZQ_OK
               : ZQ_ERR_CUDA;
  const Plan& plan = ch.plan;
  int* status = device_status_ptr();
  if (!status) return ZQ_ERR_CUDA;

  GemmParams gp{};
  gp.s_tok = s_tok;
  gp.s_grp = s_grp;
  gp.bias = static_cast<const __half*>(bias);
  gp.Y = static_cast<__half*>(Y);
  gp.acc_dbg = acc_dbg;
  gp.ws = ws;
  gp.status = status;
  gp.T = T;
  gp.N = N;
  gp.K = K;
  gp.g = g;
  gp.m_tiles = plan.m_tiles;
  gp.n_tiles = plan.n_tiles;
  gp.k_blocks = plan.k_blocks;
  gp.splits = plan.splits;
  gp.kps = plan.kps;
  gp.num_units = plan.units;
  gp.tail_start = plan.wrows ? plan.units : plan.tail_start;
  gp.tail_splits = plan.tail_splits;
  gp.tail_kb = plan.tail_kb;
  // Weight rows with several token tiles: when the weights are the larger
  // operand, let the CTAs running at the same time share a weight tile (each
  // weight tile then comes from DRAM once, the activations from L2).
  gp.n_fastest = plan.wrows && plan.n_tiles > 1 &&
                 static_cast<double>(N) * K * (w4 ? 0.5 : 1.0) > static_cast<double>(T) * K;
  if (split_partials(plan, T, N) > 0 && !ws) return ZQ_ERR_CUDA;

  // TMA descriptors: int8 activations [T][K]; weights int8 [N][K] (128B
  // swizzle, matching the MMA's K-major layout) or packed int4 [N][K/2]
  // (plain rows, unpacked into the swizzled layout by the kernel).
  const int act_rows = plan.wrows ? plan.bn : BM;
  const int w_rows = plan.wrows ? BM : (plan.pair ? plan.bn / 2 : plan.bn);
  CUtensorMap ma, mw, my;
  // INT4 weight streaming (deep ring, several K slices per stage): when K is
  // a whole number of stages, one 3-D box brings all of a stage's activation
  // slices (one TMA copy instead of plan.kps)
  gp.act3d = w4 && plan.wrows && plan.kps > 1 && K % (plan.kps * BK) == 0;
  if (gp.act3d) {
    if (!encode_tma_3d_slices(&ma, Xq, K, T, BK, act_rows, plan.kps, CU_TENSOR_MAP_SWIZZLE_128B))
      return ZQ_ERR_CUDA;
  } else if (!encode_tma_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, K, T, K, BK, act_rows,
                            CU_TENSOR_MAP_SWIZZLE_128B)) {
    return ZQ_ERR_CUDA;
  }
  if (w4) {
    // one box per stage: plan.kps K slices of 64 packed bytes per row; with
    // the TMEM operand ring (weight rows, BN <= 128) each thread reads a
    // whole 128-byte row, so those rows land 128B-swizzled (conflict-free)
    const bool tmem_a = plan.wrows && plan.bn <= 128;
    if (!encode_tma_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K / 2, N, K / 2,
                       plan.kps * (BK / 2), w_rows,
                       tmem_a ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
      return ZQ_ERR_CUDA;
  } else {
    if (!encode_tma_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, K, N, K, BK, w_rows,
                       CU_TENSOR_MAP_SWIZZLE_128B))
      return ZQ_ERR_CUDA;
  }
  if (!encode_y_map(&my, Y, T, N))
    return ZQ_ERR_CUDA;

  const int sms = num_sms();
  int grid = std::min(plan.units, sms);
  const int cap = option(ZQ_OPT_MAX_CTAS);
  if (cap > 0) grid = std::min(grid, cap);
  if (plan.pair) {  // CTA pairs: an even number of CTAs, one unit per pair at a time
    grid = 2 * std::min(plan.units, sms / 2);
    if (cap > 0) grid = std::min(grid, std::max(2, cap & ~1));
  }
  cudaError_t e;
  if (plan.pair)
    e = w4 ? dispatch_pair<true>(plan.bn, ma, mw, my, gp, grid, st)
           : dispatch_pair<false>(plan.bn, ma, mw, my, gp, grid, st);
  else if (plan.wrows)
    e = w4 ? dispatch_bn<true, true>(plan.bn, ma, mw, my, gp, grid, st)
           : dispatch_bn<true, false>(plan.bn, ma, mw, my, gp, grid, st);
  else
    e = w4 ? dispatch_bn<false, true>(plan.bn, ma, mw, my, gp, grid, st)
           : dispatch_bn<false, false>(plan.bn, ma, mw, my, gp, grid, st);
  if (e == cudaSuccess && split_partials(plan, T, N) > 0)
    e = plan.wrows ? launch_finalize(gp, st) : launch_tail_finalize(gp, plan, st);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

zq_status gemm_entry(bool w4, const int8_t* Xq, const float* s_tok, const void* Wq,
                     const float* s_grp, int g, const void* bias, int T, int N, int K, void* Y,
                     int32_t* acc_dbg, zq_stream_t stream) {
  zq_status rc = check_gemm_args(w4, Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg);
  if (rc != ZQ_OK || T == 0) return rc;
  Choice ch;
  rc = choose(w4, T, N, K, option(ZQ_OPT_SPLIT_K), &ch);
  if (rc != ZQ_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // One library workspace per device: the widened INT4 codes (N*K bytes,
  // rounded up to 256 bytes) first, when the call widens, then the split-K
  // partial sums, when its plan splits K.
  const size_t partials = ch.gemv ? 0 : split_partials(ch.plan, T, N);
  const size_t wide_ints = ch.widen ? (static_cast<size_t>(N) * K + 255) / 256 * 64 : 0;
  int32_t* ws = nullptr;
  if (partials > 0 || wide_ints > 0) {
    rc = ensure_workspace(wide_ints + partials, true, st, &ws);
    if (rc != ZQ_OK) return rc;
  }
  if (ch.widen) {
    const size_t n16 = static_cast<size_t>(N) * (K / 2) / 16;
    const int blocks = static_cast<int>(std::min<size_t>((n16 + 255) / 256, 8 * num_sms()));
    // (8 resident CTAs of 256 threads per SM, each thread kWidenUnroll
    // chunks in flight)
    if (launch_pdl(widen_w4_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, st,
                   static_cast<const uint4*>(Wq), reinterpret_cast<uint4*>(ws), n16) != cudaSuccess)
      return ZQ_ERR_CUDA;
    return launch_choice(false, ch, Xq, s_tok, ws, s_grp, g, bias, T, N, K, Y, acc_dbg,
                         partials > 0 ? ws + wide_ints : nullptr, st);
  }
  return launch_choice(w4, ch, Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg, ws, st);
}

}  // namespace
}  // namespace zq

extern "C" zq_status zq_widen_int4_weights(const uint8_t* Wq4, int N, int K, int8_t* Wq8,
                                           zq_stream_t stream) {
  using namespace zq;
  if (N < 1 || K < 32 || K % 32 != 0) return ZQ_ERR_SHAPE;
  if (!Wq4 || !Wq8) return ZQ_ERR_NULL;
  if (!aligned16(Wq4) || !aligned16(Wq8)) return ZQ_ERR_ALIGN;
  const size_t n16 = static_cast<size_t>(N) * (K / 2) / 16;
  const int blocks = static_cast<int>(std::min<size_t>((n16 + 255) / 256, 8 * num_sms()));
  if (launch_pdl(widen_w4_kernel, dim3(std::max(blocks, 1)), dim3(256), 0,
                 reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(Wq4),
                 reinterpret_cast<uint4*>(Wq8), n16) != cudaSuccess)
    return ZQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

extern "C" zq_status zq_workspace_reserve(unsigned long long bytes) {
  int32_t* p = nullptr;
  if (bytes == 0) return ZQ_OK;
  return zq::ensure_workspace((bytes + 3) / 4, false, nullptr, &p);
}

extern "C" zq_status zq_gemm_w8a8(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                                  const float* s_grp, int g, const void* bias, int T, int N,
                                  int K, void* Y, int32_t* acc_dbg, zq_stream_t stream) {
  return zq::gemm_entry(false, Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg, stream);
}

extern "C" zq_status zq_gemm_w4a8(const int8_t* Xq, const float* s_tok, const uint8_t* Wq4,
                                  const float* s_grp, int g, const void* bias, int T, int N,
                                  int K, void* Y, int32_t* acc_dbg, zq_stream_t stream) {
  return zq::gemm_entry(true, Xq, s_tok, Wq4, s_grp, g, bias, T, N, K, Y, acc_dbg, stream);
}

// ----------------------------------------------------------------------------
// Allocation-free variant of zq_gemm_w8a8.
//
// The split-K reduction of the weight-streaming tiling needs scratch memory
// (one int32 partial-sum slice per K split).
// zq_gemm_w8a8 allocates that lazily with cudaMalloc.  Some callers cannot
// let a library allocate: a serving runtime that owns the whole device
// memory pool, a process whose memory budget is fixed up front, or code that
// must never trigger the device-wide synchronisation cudaMalloc/cudaFree can
// imply.  This variant takes its scratch from a fixed array in device memory
// that exists from library load until process exit on every GPU that loads
// the library.
namespace zq {
namespace {

constexpr size_t kNoAllocPartialInts = (8u << 20) / sizeof(int32_t);  // 8 MiB of partial sums

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocPartialInts];

std::mutex g_noalloc_mu;
int32_t* g_noalloc_ptr[64] = {};

// Device address of the fixed scratch on the current device.  Host code
// cannot use the array's name as a device pointer; the address is looked up
// once per device, with that device current.
cudaError_t noalloc_scratch(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace zq

extern "C" zq_status zq_gemm_w8a8_noalloc(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                                          const float* s_grp, int g, const void* bias, int T,
                                          int N, int K, void* Y, int32_t* acc_dbg,
                                          zq_stream_t stream) {
  using namespace zq;
  zq_status rc = check_gemm_args(false, Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg);
  if (rc != ZQ_OK || T == 0) return rc;
  // The same choice of kernel and plan as zq_gemm_w8a8.  When its K splits
  // would need more partial sums than the fixed array holds, plan again with
  // as many splits as fit (one split needs no scratch at all); only a split
  // count forced through ZQ_OPT_SPLIT_K that does not fit is refused.
  const int forced_split = option(ZQ_OPT_SPLIT_K);
  Choice ch;
  rc = choose(false, T, N, K, forced_split, &ch);
  if (rc != ZQ_OK) return rc;
  if (!ch.gemv && !ch.plan.wrows && split_partials(ch.plan, T, N) > kNoAllocPartialInts) {
    // a token-row plan whose last-wave split does not fit: plan without it
    rc = choose(false, T, N, K, forced_split, &ch, false);
    if (rc != ZQ_OK) return rc;
  }
  if (!ch.gemv && split_partials(ch.plan, T, N) > kNoAllocPartialInts) {
    if (forced_split > 0) return ZQ_ERR_SHAPE;
    const size_t fit = kNoAllocPartialInts / (static_cast<size_t>(T) * N);
    rc = choose(false, T, N, K, static_cast<int>(std::max<size_t>(1, std::min<size_t>(fit, 32))),
                &ch);
    if (rc != ZQ_OK) return rc;
    if (split_partials(ch.plan, T, N) > kNoAllocPartialInts) return ZQ_ERR_SHAPE;
  }
  int32_t* scratch = nullptr;
  if (!ch.gemv && split_partials(ch.plan, T, N) > 0) {
    if (noalloc_scratch(&scratch) != cudaSuccess) return ZQ_ERR_CUDA;
    // every partial sum the finalisation reads is written by this call
  }
  return launch_choice(false, ch, Xq, s_tok, Wq, s_grp, g, bias, T, N, K, Y, acc_dbg, scratch,
                       reinterpret_cast<cudaStream_t>(stream));
}
