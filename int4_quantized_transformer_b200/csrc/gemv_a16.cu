// gemv_a16.cu -- the FP16-activation quantized linear layer (W8A16, W4A16)
// for a handful of tokens (T <= 4) on CUDA cores: a matrix-vector product
// streamed straight from HBM.
//
// Same arithmetic as gemm_a16.cu (the ZeroQuant summary page's W8A16 and
// W4/8A16 configurations): acc[t][o] = sum_k x[t][k] * q[o][k], every
// product exact and summed in fp32 (here by fma, in this kernel's order),
// then y = fp16(f32(acc * s_grp[group(o)]) + f32(bias[o])).
//
// At T <= 4 every weight byte meets at most four activations.  Each warp
// streams whole weight rows with coalesced 16-byte loads; codes become exact
// fp32 values with one byte permute and one add each (the code's sign bit
// flipped is placed as the low byte of the float 2^23, giving 2^23 + c + 128
// -- or 2^23 + c + 8 for a nibble -- and subtracting that offset leaves c);
// the activations are converted once per k and reused by every row of the
// warp.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>

#include "zq_internal.h"
#include "zq_ptx.cuh"

namespace zq {
namespace {

constexpr int kA16Threads = 256;  // 8 warps per CTA

template <int TT>
struct A16GemvShape {
  static constexpr int ROWS = TT == 1 ? 2 : (TT == 2 ? 4 : 8);
  static constexpr int UNROLL = TT == 1 ? 3 : (TT == 2 ? 2 : 1);
};

__device__ __forceinline__ int a16v_group_of(int o, int N, int g) {
  const unsigned long long prod = static_cast<unsigned long long>(o) * static_cast<unsigned>(g);
  if (prod < (1ull << 32))
    return static_cast<int>(static_cast<unsigned>(prod) / static_cast<unsigned>(N));
  return static_cast<int>(prod / static_cast<unsigned>(N));
}

// Byte i of u (0..255) as the float 2^23 + u_i.
template <int I>
__device__ __forceinline__ float byte_as_float(uint32_t u) {
  return __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u | I));
}

// Eight codes k = 0..7 of one group of eight -> exact floats.
// BITS = 8: two words (k 0..3, k 4..7), one int8 code per byte.
// BITS = 4: one word; byte i holds k = i (low nibble) and k = 4 + i (high).
template <int BITS>
__device__ __forceinline__ void codes8(uint32_t w0, uint32_t w1, float (&q)[8]) {
  if constexpr (BITS == 8) {
    const uint32_t a = w0 ^ 0x80808080u, b = w1 ^ 0x80808080u;
    constexpr float off = 8388608.0f + 128.0f;
    q[0] = byte_as_float<0>(a) - off;
    q[1] = byte_as_float<1>(a) - off;
    q[2] = byte_as_float<2>(a) - off;
    q[3] = byte_as_float<3>(a) - off;
    q[4] = byte_as_float<0>(b) - off;
    q[5] = byte_as_float<1>(b) - off;
    q[6] = byte_as_float<2>(b) - off;
    q[7] = byte_as_float<3>(b) - off;
  } else {
    const uint32_t u = w0 ^ 0x88888888u;
    const uint32_t lo = u & 0x0F0F0F0Fu, hi = (u >> 4) & 0x0F0F0F0Fu;
    constexpr float off = 8388608.0f + 8.0f;
    q[0] = byte_as_float<0>(lo) - off;
    q[1] = byte_as_float<1>(lo) - off;
    q[2] = byte_as_float<2>(lo) - off;
    q[3] = byte_as_float<3>(lo) - off;
    q[4] = byte_as_float<0>(hi) - off;
    q[5] = byte_as_float<1>(hi) - off;
    q[6] = byte_as_float<2>(hi) - off;
    q[7] = byte_as_float<3>(hi) - off;
  }
}

// A 16-byte weight chunk holds KPC = 16 (int8) or 32 (int4) consecutive k.
// A CTA of 8 warps takes 8/KS row groups of ROWS rows; the KS warps of a row
// group split the row's chunks into KS contiguous ranges and add their fp32
// partial sums through shared memory.
template <int BITS, int TT>
__global__ void __launch_bounds__(kA16Threads)
    gemv_a16_kernel(const __half* __restrict__ X, const uint8_t* __restrict__ W,
                    const float* __restrict__ s_grp, int g, const __half* __restrict__ bias,
                    int T, int N, int K, int KS, __half* __restrict__ Y,
                    float* __restrict__ acc_dbg) {
  constexpr int KPC = BITS == 4 ? 32 : 16;
  constexpr int kRows = A16GemvShape<TT>::ROWS;
  constexpr int kUnroll = A16GemvShape<TT>::UNROLL;
  constexpr int kWarps = kA16Threads / 32;
  __shared__ float red[kWarps][kRows * TT];
  // X may be written by the previous kernel of the stream
  grid_dependency_wait();
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int rg = warp / KS, ks = warp % KS;
  const int groups = kWarps / KS;
  const int chunks = K / KPC;
  const int per = (chunks + KS - 1) / KS;
  const int cbeg = ks * per, cend = min(chunks, cbeg + per);
  const size_t row_bytes = static_cast<size_t>(K) * BITS / 8;

  // the loop bound depends only on blockIdx: the __syncthreads are uniform
  for (int ob = blockIdx.x * groups * kRows; ob < N; ob += gridDim.x * groups * kRows) {
    const int o0 = ob + rg * kRows;
    float acc[kRows][TT];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[r][t] = 0.0f;

    for (int c0 = cbeg + lane; c0 < cend; c0 += 32 * kUnroll) {
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
        // groups of eight k: a W8 chunk has two (words 0-1, 2-3), a W4 chunk
        // four (one word each)
#pragma unroll
        for (int e = 0; e < KPC / 8; ++e) {
          float xf[TT][8];
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            if (t < T) {
              const uint4 xv = __ldg(reinterpret_cast<const uint4*>(
                  X + static_cast<size_t>(t) * K + static_cast<size_t>(c) * KPC + 8 * e));
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xw[i]));
                xf[t][2 * i] = f.x;
                xf[t][2 * i + 1] = f.y;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) xf[t][i] = 0.0f;
            }
          }
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            const uint32_t pw[4] = {w[u][r].x, w[u][r].y, w[u][r].z, w[u][r].w};
            float q[8];
            if constexpr (BITS == 8)
              codes8<8>(pw[2 * e], pw[2 * e + 1], q);
            else
              codes8<4>(pw[e], 0u, q);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              float a = acc[r][t];
#pragma unroll
              for (int i = 0; i < 8; ++i) a = __fmaf_rn(xf[t][i], q[i], a);
              acc[r][t] = a;
            }
          }
        }
      }
    }

    // fp32 sums across the warp, then across the KS warps of the row group
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        float v = acc[r][t];
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
        float v = 0.0f;
        for (int q = 0; q < KS; ++q) v += red[warp + q][lane];
        const size_t idx = static_cast<size_t>(t) * N + o;
        const float y = __fadd_rn(__fmul_rn(v, __ldg(s_grp + a16v_group_of(o, N, g))),
                                  bias ? __half2float(bias[o]) : 0.0f);
        Y[idx] = __float2half_rn(y);
        if (acc_dbg) acc_dbg[idx] = v;
      }
    }
    __syncthreads();  // red is reused by the next row block
  }
}

template <int BITS, int TT>
cudaError_t launch_a16_tt(const void* X, const void* W, const float* s_grp, int g,
                          const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                          int max_ctas, cudaStream_t st) {
  static std::atomic<int> resident[64];  // per device; a repeated query is harmless
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && resident[dev].load(std::memory_order_acquire) == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_a16_kernel<BITS, TT>,
                                                      kA16Threads, 0) != cudaSuccess ||
        per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    resident[dev].store(per_sm, std::memory_order_release);
  }
  const int per_sm = (dev >= 0 && dev < 64) ? resident[dev].load() : 1;
  constexpr int kRows = A16GemvShape<TT>::ROWS;
  constexpr int round = 32 * A16GemvShape<TT>::UNROLL;
  const int chunks = K / (BITS == 4 ? 32 : 16);
  int ks = 1;
  while (ks < kA16Threads / 32 && chunks / (2 * ks) >= 2 * round) ks *= 2;
  const int rows_per_cta = (kA16Threads / 32 / ks) * kRows;
  int grid = std::min((N + rows_per_cta - 1) / rows_per_cta, per_sm * num_sms());
  if (max_ctas > 0) grid = std::min(grid, max_ctas);
  grid = std::max(grid, 1);
  return launch_pdl(gemv_a16_kernel<BITS, TT>, dim3(grid), dim3(kA16Threads), 0, st,
                    static_cast<const __half*>(X), static_cast<const uint8_t*>(W), s_grp, g,
                    static_cast<const __half*>(bias), T, N, K, ks, static_cast<__half*>(Y),
                    acc_dbg);
}

}  // namespace

cudaError_t launch_gemv_a16(int bits, const void* X, const void* W, const float* s_grp, int g,
                            const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                            int max_ctas, cudaStream_t st) {
  if (T < 1 || T > kGemvA16MaxTokens) return cudaErrorInvalidValue;
  if (bits == 4) {
    if (T == 1) return launch_a16_tt<4, 1>(X, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
    if (T == 2) return launch_a16_tt<4, 2>(X, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
    return launch_a16_tt<4, 4>(X, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
  }
  if (T == 1) return launch_a16_tt<8, 1>(X, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
  if (T == 2) return launch_a16_tt<8, 2>(X, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
  return launch_a16_tt<8, 4>(X, W, s_grp, g, bias, T, N, K, Y, acc_dbg, max_ctas, st);
}

}  // namespace zq
