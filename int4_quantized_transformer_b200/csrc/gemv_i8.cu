// gemv_i8.cu -- the quantized linear layer for a handful of tokens (T <= 4)
// on CUDA cores: a matrix-vector product streamed straight from HBM.
//
// ZeroQuant (arXiv 2206.01861), Sec. 3.4 "Scheduling for different batch
// sizes": small batches are memory-bound and get their own kernel.  At
// T <= 4 the weights are read once and every weight byte meets at most four
// activations, so the work is a memory-bound GEMV.  On the tensor-core path
// the weights would make several trips through shared memory (TMA write,
// INT4 widening, MMA operand read); here each warp streams whole weight rows
// with coalesced 16-byte loads, widens INT4 codes in registers and
// accumulates with dp4a (exact int32), so the only per-byte cost besides HBM
// is a few integer instructions.
//
// The arithmetic is the one of the GEMM epilogue ("Dequantization fused into
// the GEMM epilogue"): acc[t][o] = sum_k Xq[t][k] * Wq[o][k] in int32, then
// y = fp16(((f32(acc) * s_tok[t]) * s_grp[group(o)]) + f32(bias[o])).
// INT4 codes are widened to int8 as codes*16 (two logic ops per eight codes,
// the packed layout of zq_gemm_w4a8) and the int32 sum is divided by 16
// exactly at the end.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>

#include "zq_internal.h"
#include "zq_ptx.cuh"

namespace zq {
namespace {

constexpr int kGemvThreads = 256;  // 8 warps per CTA

// Weight rows a warp streams together, and 16-byte chunks per row and lane
// loaded before any is used.  More tokens reuse each activation load across
// more rows (the activation reads from L1 would otherwise bound T = 4);
// fewer tokens keep more chunks of fewer rows in flight.
template <int TT>
struct GemvShape {
  static constexpr int ROWS = TT == 1 ? 2 : (TT == 2 ? 4 : 8);
  static constexpr int UNROLL = TT == 1 ? 3 : (TT == 2 ? 2 : 1);
};

__device__ __forceinline__ int group_of_row(int o, int N, int g) {
  const unsigned long long prod = static_cast<unsigned long long>(o) * static_cast<unsigned>(g);
  if (prod < (1ull << 32))
    return static_cast<int>(static_cast<unsigned>(prod) / static_cast<unsigned>(N));
  return static_cast<int>(prod / static_cast<unsigned>(N));
}

// BITS = 8: a 16-byte chunk of a weight row holds 16 int8 codes (k = 16c ..
// 16c+15).  BITS = 4: it holds 32 packed codes (k = 32c .. 32c+31); in each
// 32-bit word, byte i carries k = 8m+i in its low nibble and k = 8m+4+i in
// its high nibble.
//
// A CTA of 8 warps takes 8/KS row groups of ROWS rows; the KS warps of a row
// group split the row's chunks into KS contiguous ranges, and their int32
// partial sums are added (exactly) through shared memory.  KS > 1 keeps the
// GPU full when N is small and K large.
template <int BITS, int TT>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_i8_kernel(const int8_t* __restrict__ Xq, const float* __restrict__ s_tok,
                   const uint8_t* __restrict__ W, const float* __restrict__ s_grp, int g,
                   const __half* __restrict__ bias, int T, int N, int K, int KS,
                   __half* __restrict__ Y, int32_t* __restrict__ acc_dbg) {
  constexpr int KPC = BITS == 4 ? 32 : 16;  // k values per 16-byte weight chunk
  constexpr int kRows = GemvShape<TT>::ROWS;
  constexpr int kUnroll = GemvShape<TT>::UNROLL;
  constexpr int kWarps = kGemvThreads / 32;
  __shared__ int red[kWarps][kRows * TT];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int rg = warp / KS, ks = warp % KS;  // row group, K range
  const int groups = kWarps / KS;
  const int chunks = K / KPC;
  const int per = (chunks + KS - 1) / KS;
  const int cbeg = ks * per, cend = min(chunks, cbeg + per);
  const size_t row_bytes = static_cast<size_t>(K) * BITS / 8;
  // The CTA's first block of weight rows (contiguous) goes to L2 before the
  // wait for the previous kernel, so the HBM stream starts while it runs
  // (only L2 is touched: the weights cannot be read stale).
  if (threadIdx.x == 0) {
    const int r0 = blockIdx.x * groups * kRows;
    const int nr = min(groups * kRows, N - r0);
    if (nr > 0) {
      const char* base = reinterpret_cast<const char*>(W) + static_cast<size_t>(r0) * row_bytes;
      size_t left = static_cast<size_t>(nr) * row_bytes;
      while (left > 0) {  // row_bytes is a multiple of 16
        const uint32_t n = static_cast<uint32_t>(left < (1u << 20) ? left : (1u << 20));
        bulk_prefetch_l2(base, n);
        base += n;
        left -= n;
      }
    }
  }
  // Xq and s_tok may be written by the previous kernel of the stream
  grid_dependency_wait();
  grid_launch_dependents();

  // every warp of the CTA runs the same number of iterations (the bound
  // depends only on blockIdx), so the __syncthreads below are uniform
  for (int ob = blockIdx.x * groups * kRows; ob < N; ob += gridDim.x * groups * kRows) {
    const int o0 = ob + rg * kRows;
    int acc[kRows][TT];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[r][t] = 0;

    for (int c0 = cbeg + lane; c0 < cend; c0 += 32 * kUnroll) {
      // issue every weight load of this round before using any of them
      uint4 w[kUnroll][kRows];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = c0 + 32 * u;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          w[u][r] = make_uint4(0u, 0u, 0u, 0u);
          if (c < cend && o0 + r < N)
            w[u][r] = __ldcs(
                reinterpret_cast<const uint4*>(W + static_cast<size_t>(o0 + r) * row_bytes) + c);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = c0 + 32 * u;
        if (c >= cend) break;
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          if (t >= T) break;
          const int4* xp = reinterpret_cast<const int4*>(Xq + static_cast<size_t>(t) * K +
                                                         static_cast<size_t>(c) * KPC);
          if constexpr (BITS == 4) {
            const int4 xa = __ldg(xp), xb = __ldg(xp + 1);  // k = 32c .. 32c+31
            const int xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
              const uint32_t pw[4] = {w[u][r].x, w[u][r].y, w[u][r].z, w[u][r].w};
              int a = acc[r][t];
#pragma unroll
              for (int m = 0; m < 4; ++m) {
                // word m covers k = 8m .. 8m+7 of the chunk: widened as codes*16
                const int lo = static_cast<int>((pw[m] << 4) & 0xF0F0F0F0u);  // k = 8m .. 8m+3
                const int hi = static_cast<int>(pw[m] & 0xF0F0F0F0u);         // k = 8m+4 .. 8m+7
                a = __dp4a(lo, xw[2 * m], a);
                a = __dp4a(hi, xw[2 * m + 1], a);
              }
              acc[r][t] = a;
            }
          } else {
            const int4 xa = __ldg(xp);  // k = 16c .. 16c+15
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
              int a = acc[r][t];
              a = __dp4a(static_cast<int>(w[u][r].x), xa.x, a);
              a = __dp4a(static_cast<int>(w[u][r].y), xa.y, a);
              a = __dp4a(static_cast<int>(w[u][r].z), xa.z, a);
              a = __dp4a(static_cast<int>(w[u][r].w), xa.w, a);
              acc[r][t] = a;
            }
          }
        }
      }
    }

    // exact int32 sums: across the warp, then across the KS warps of the
    // row group; lane j of the group's first warp finishes output j
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        int v = acc[r][t];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) red[warp][r * TT + t] = v;
      }
    }
    __syncthreads();
    if (ks == 0 && lane < kRows * TT) {
      const int r = lane / TT, t = lane % TT;
      const int o = o0 + r;
      if (o < N && t < T) {
        int v = 0;
        for (int q = 0; q < KS; ++q) v += red[warp + q][lane];
        const int a = BITS == 4 ? (v >> 4) : v;  // INT4 codes were widened as codes*16
        const size_t idx = static_cast<size_t>(t) * N + o;
        float y = __fmul_rn(__int2float_rn(a), __ldg(s_tok + t));
        y = __fadd_rn(__fmul_rn(y, __ldg(s_grp + group_of_row(o, N, g))),
                      bias ? __half2float(bias[o]) : 0.0f);
        Y[idx] = __float2half_rn(y);
        if (acc_dbg) acc_dbg[idx] = a;
      }
    }
    __syncthreads();  // red is reused by the next row block
  }
}

// One launch: as many CTAs as are resident at once (the row loop is
// grid-strided, so a second, serial wave of CTAs would only add a tail), or
// fewer when there are fewer row blocks.  KS, the warps that share a row
// group, grows with K until each warp keeps at least two rounds of chunks.
template <int BITS, int TT>
cudaError_t launch_tt(const int8_t* Xq, const float* s_tok, const void* W, const float* s_grp,
                      int g, const void* bias, int T, int N, int K, void* Y, int32_t* acc_dbg,
                      int max_ctas, cudaStream_t st) {
  static std::atomic<int> resident[64];  // per device; a repeated query is harmless
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && resident[dev].load(std::memory_order_acquire) == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_i8_kernel<BITS, TT>,
                                                      kGemvThreads, 0) != cudaSuccess ||
        per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    resident[dev].store(per_sm, std::memory_order_release);
  }
  const int per_sm = (dev >= 0 && dev < 64) ? resident[dev].load() : 1;
  constexpr int kRows = GemvShape<TT>::ROWS;
  constexpr int round = 32 * GemvShape<TT>::UNROLL;
  const int chunks = K / (BITS == 4 ? 32 : 16);
  int ks = 1;
  while (ks < kGemvThreads / 32 && chunks / (2 * ks) >= 2 * round) ks *= 2;
  const int rows_per_cta = (kGemvThreads / 32 / ks) * kRows;
  int grid = std::min((N + rows_per_cta - 1) / rows_per_cta, per_sm * num_sms());
  if (max_ctas > 0) grid = std::min(grid, max_ctas);
  grid = std::max(grid, 1);
  return launch_pdl(gemv_i8_kernel<BITS, TT>, dim3(grid), dim3(kGemvThreads), 0, st, Xq, s_tok,
                    static_cast<const uint8_t*>(W), s_grp, g, static_cast<const __half*>(bias), T,
                    N, K, ks, static_cast<__half*>(Y), acc_dbg);
}

}  // namespace

cudaError_t launch_gemv_i8(int bits, const int8_t* Xq, const float* s_tok, const void* W,
                           const float* s_grp, int g, const void* bias, int T, int N, int K,
                           void* Y, int32_t* acc_dbg, int max_ctas, cudaStream_t st) {
  if (T < 1 || T > kGemvMaxTokens) return cudaErrorInvalidValue;
  if (bits == 4) {
    if (T == 1) return launch_tt<4, 1>(Xq, s_tok, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
    if (T == 2) return launch_tt<4, 2>(Xq, s_tok, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
    return launch_tt<4, 4>(Xq, s_tok, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
  }
  if (T == 1) return launch_tt<8, 1>(Xq, s_tok, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
  if (T == 2) return launch_tt<8, 2>(Xq, s_tok, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
  return launch_tt<8, 4>(Xq, s_tok, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
}

}  // namespace zq
