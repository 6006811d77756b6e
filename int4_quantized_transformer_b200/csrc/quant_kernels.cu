// quant_kernels.cu -- the two HBM-bound quantizers of the fused quantized
// linear layer (ZeroQuant, arXiv 2206.01861, Sec. 3.4):
//
//  * ln_quant: fused LayerNorm + token-wise dynamic INT8 quantization
//    ("Kernel fusion for token-wise activation quantization", Fig. 2 right):
//    each row is read once into registers with 128-bit loads, its exact
//    statistics, fp16 LayerNorm output and absmax are reduced with warp
//    shuffles (plus shared memory when several warps share a row), and only
//    the int8 row and its scale are written back.
//  * wquant: group-wise weight quantization ("Group-wise Weight
//    Quantization", Eq. 2), one CTA per group of contiguous output rows,
//    with optional packing of two signed INT4 codes per byte (of each eight
//    consecutive k, byte i holds k = i and k = 4 + i).
//
// Every floating-point step uses an explicit round-to-nearest intrinsic so
// that the compiler cannot contract it into an FMA: results are bit-exact
// with respect to the op-by-op definition in include/zq.h.
#include <cuda_fp16.h>

#include "zq_internal.h"
#include "zq_ptx.cuh"

namespace zq {
namespace {

// Round-half-to-even of |v| < 2^22 to an integer, returned in the low byte
// of the result: adding 1.5*2^23 leaves an fp32 whose unit in the last
// place is 1, so the IEEE round-to-nearest-even addition performs the
// rounding and the integer appears in the low mantissa bits (the classic
// "magic number" conversion).
__device__ __forceinline__ uint32_t rne_low_byte(float v) {
  return __float_as_uint(__fadd_rn(v, 12582912.0f));
}

// Eq. 2 for one element once the per-set scale is known: clamp to
// [-qmax, qmax] (clamping before or after rounding is the same for integer
// bounds), round half to even.  Returns the code in the low byte.
__device__ __forceinline__ uint32_t quant_code(float y, float inv, float qmax) {
  float v = __fmul_rn(y, inv);
  v = fminf(fmaxf(v, -qmax), qmax);
  return rne_low_byte(v);
}

// Token quantization of one element: as quant_code with qmax = 127, without
// the clamp, which cannot bind here: amax = max|y| over the row and
// inv = fp32(127/amax), so |y*inv| <= 127*(1+2^-24)^2 and its rounding to the
// nearest integer is at most 127.
__device__ __forceinline__ uint32_t token_code(float y, float inv) {
  return rne_low_byte(__fmul_rn(y, inv));
}

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  uint32_t lo = __byte_perm(a, b, 0x0040);
  uint32_t hi = __byte_perm(c, d, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// --------------------------------------------------------------- ln_quant

struct RowSums {
  long long s1;            // sum of a = x * 2^24 (an integer for every finite fp16 x)
  unsigned long long p;    // sum of ah^2    } with a = ah*2^20 + al, ah = floor(x*16),
  long long q;             // sum of ah*al   } al in [0, 2^20): a^2 = p*2^40 + q*2^21 + r
  unsigned long long r;    // sum of al^2    }
};

// Per-thread partial sums: a thread adds at most 32 elements, so sum(ah) and
// sum(al) stay below 2^26 in magnitude and fit 32-bit integers.
struct ThreadSums {
  int s1h, s1l;
  unsigned long long p, r;
  long long q;
};

// Adds one fp16 value x (already converted to fp32, exactly) to the exact
// sums.  a = x*2^24 = ah*2^20 + al with ah = floor(x*16) (|ah| <= 2^20) and
// al = (x*16 - ah)*2^20 in [0, 2^20).  Both come from the fp32 "magic
// number" technique: adding 1.5*2^23 with rounding toward zero leaves
// floor(v) in the low mantissa bits (|v| < 2^20, the sum stays in
// [2^23, 2^24) where the spacing is 1), and the remaining fraction is an
// exact multiple of 2^-20.
__device__ __forceinline__ void add_exact(ThreadSums& s, float x) {
  const float v = __fmul_rn(x, 16.0f);                       // exact, |v| < 2^20
  const float t = __fadd_rz(v, 12582912.0f);                 // 1.5*2^23 + floor(v)
  const int ah = static_cast<int>(__float_as_uint(t) - 0x4B400000u);
  const float fr = __fsub_rn(v, __fsub_rn(t, 12582912.0f));  // v - floor(v), exact
  const int al = static_cast<int>(__float_as_uint(__fmaf_rn(fr, 1048576.0f, 8388608.0f)) -
                                  0x4B000000u);
  s.s1h += ah;
  s.s1l += al;
  s.p += static_cast<unsigned long long>(static_cast<long long>(ah) * ah);
  s.q += static_cast<long long>(ah) * al;
  s.r += static_cast<unsigned long long>(al) * static_cast<unsigned int>(al);
}

__device__ __forceinline__ void warp_sum(RowSums& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s.s1 += __shfl_xor_sync(0xffffffffu, s.s1, o);
    s.p += __shfl_xor_sync(0xffffffffu, s.p, o);
    s.q += __shfl_xor_sync(0xffffffffu, s.q, o);
    s.r += __shfl_xor_sync(0xffffffffu, s.r, o);
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// mean and rstd from the exact sums, c1 = 2^-24/K and c2 = 2^-48/K (fp64,
// computed on the host): mean = S1*c1, E[x^2] = S2*c2 with S2 taken to
// fp64 as hi*2^64 + lo, var = max(E[x^2] - mean^2, 0) (biased) in fp64, then
// rstd = 1/sqrt(fp32(var) + eps) in fp32.
__device__ __forceinline__ void row_stats(const RowSums& s, double c1, double c2, float eps,
                                          float& mean, float& rstd) {
  const __int128 s2s = (static_cast<__int128>(s.p) << 40) + (static_cast<__int128>(s.q) << 21) +
                       static_cast<__int128>(s.r);
  const unsigned __int128 s2 = static_cast<unsigned __int128>(s2s);  // a sum of squares: >= 0
  const unsigned long long hi = static_cast<unsigned long long>(s2 >> 64);
  const unsigned long long lo = static_cast<unsigned long long>(s2);
  const double mean_d = __dmul_rn(__ll2double_rn(s.s1), c1);
  const double e2 =
      __dmul_rn(__dadd_rn(__dmul_rn(__ull2double_rn(hi), 0x1p64), __ull2double_rn(lo)), c2);
  double var = __dsub_rn(e2, __dmul_rn(mean_d, mean_d));
  if (var < 0.0) var = 0.0;
  const float r = __fsqrt_rn(__fadd_rn(__double2float_rn(var), eps));
  rstd = __fdiv_rn(1.0f, r);
  mean = __double2float_rn(mean_d);
}

// W warps per row, VPT 16-byte vectors (8 halves) per thread.  Blocks hold
// RPB = max(1, 8/W) rows; every thread runs the same number of row
// iterations so block-wide barriers stay uniform.  gamma/beta are re-read
// per row (they stay in L1) to keep registers low and occupancy high.
template <int W, int VPT>
__global__ void __launch_bounds__((W >= 8 ? W : 8) * 32, (W >= 8 ? 2048 / (W * 32) : 8) / 2)
    ln_quant_kernel(const __half* __restrict__ X, const __half* __restrict__ gamma,
                    const __half* __restrict__ beta, int T, int K, float eps, double c1,
                    double c2, int8_t* __restrict__ Xq, float* __restrict__ s_tok,
                    __half* __restrict__ Y_ln) {
  constexpr int RT = 32 * W;                // threads per row
  constexpr int RPB = W >= 8 ? 1 : 8 / W;   // rows per block
  __shared__ RowSums red_s[RPB][W];
  __shared__ float red_m[RPB][W];

  const int slot = threadIdx.x / RT;
  const int j = threadIdx.x % RT;
  const int warp_in_row = j / 32;
  const int lane = threadIdx.x & 31;
  const int nvec = K / 8;
  const bool ln = gamma != nullptr;
  grid_dependency_wait();
  grid_launch_dependents();

  const int rows_per_iter = gridDim.x * RPB;
  const int iters = (T + rows_per_iter - 1) / rows_per_iter;
  for (int it = 0; it < iters; ++it) {
    const int row = (it * gridDim.x + blockIdx.x) * RPB + slot;
    const bool valid = row < T;
    const __half* xr = X + static_cast<size_t>(row) * K;

    uint4 x4[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      int v = j + i * RT;
      x4[i] = make_uint4(0, 0, 0, 0);
      if (valid && v < nvec) x4[i] = __ldcs(reinterpret_cast<const uint4*>(xr) + v);
    }

    if (ln) {
      ThreadSums ts = {0, 0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const __half2* h = reinterpret_cast<const __half2*>(&x4[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(h[e]);
          add_exact(ts, f.x);
          add_exact(ts, f.y);
        }
      }
      RowSums s;
      s.s1 = static_cast<long long>(ts.s1h) * 1048576 + ts.s1l;
      s.p = ts.p;
      s.q = ts.q;
      s.r = ts.r;
      warp_sum(s);
      if (W > 1) {
        if (lane == 0) red_s[slot][warp_in_row] = s;
        __syncthreads();
        s = red_s[slot][0];
#pragma unroll
        for (int w = 1; w < W; ++w) {
          RowSums t = red_s[slot][w];
          s.s1 += t.s1;
          s.p += t.p;
          s.q += t.q;
          s.r += t.r;
        }
      }
      // One lane does the fp64 row arithmetic; the warp gets it by shuffle.
      float mean = 0.0f, rstd = 0.0f;
      if (lane == 0) row_stats(s, c1, c2, eps, mean, rstd);
      mean = __shfl_sync(0xffffffffu, mean, 0);
      rstd = __shfl_sync(0xffffffffu, rstd, 0);
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int v = j + i * RT;
        if (v < nvec) {
          const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
          const uint4 b4 = beta ? __ldg(reinterpret_cast<const uint4*>(beta) + v)
                                : make_uint4(0, 0, 0, 0);
          __half2* h = reinterpret_cast<__half2*>(&x4[i]);
          const __half2* gm = reinterpret_cast<const __half2*>(&g4);
          const __half2* bt = reinterpret_cast<const __half2*>(&b4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xf = __half22float2(h[e]);
            const float2 gf = __half22float2(gm[e]);
            const float2 bf = __half22float2(bt[e]);
            const float y0 = __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(xf.x, mean), rstd), gf.x), bf.x);
            const float y1 = __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(xf.y, mean), rstd), gf.y), bf.y);
            h[e] = __halves2half2(__float2half_rn(y0), __float2half_rn(y1));
          }
        }
      }
    }

    __half2 m2 = __float2half2_rn(0.0f);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const __half2* h = reinterpret_cast<const __half2*>(&x4[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) m2 = __hmax2(m2, __habs2(h[e]));
    }
    float amax = fmaxf(__low2float(m2), __high2float(m2));
    amax = warp_max(amax);
    if (W > 1) {
      if (lane == 0) red_m[slot][warp_in_row] = amax;
      __syncthreads();
#pragma unroll
      for (int w = 0; w < W; ++w) amax = fmaxf(amax, red_m[slot][w]);
      __syncthreads();  // red_s / red_m are reused by the next row
    }
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (valid) {
      if (j == 0) s_tok[row] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
      int8_t* qr = Xq + static_cast<size_t>(row) * K;
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        int v = j + i * RT;
        if (v < nvec) {
          const __half2* h = reinterpret_cast<const __half2*>(&x4[i]);
          uint32_t c[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            c[2 * e] = token_code(f.x, inv);
            c[2 * e + 1] = token_code(f.y, inv);
          }
          uint2 out;
          out.x = pack4(c[0], c[1], c[2], c[3]);
          out.y = pack4(c[4], c[5], c[6], c[7]);
          __stcs(reinterpret_cast<uint2*>(qr) + v, out);
          if (Y_ln) reinterpret_cast<uint4*>(Y_ln + static_cast<size_t>(row) * K)[v] = x4[i];
        }
      }
    }
  }
}

template <int W, int VPT>
cudaError_t launch_ln(const __half* X, const __half* g, const __half* b, int T, int K, float eps,
                      int8_t* Xq, float* s, __half* Y, cudaStream_t st) {
  constexpr int RPB = W >= 8 ? 1 : 8 / W;
  constexpr int threads = RPB * 32 * W;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, ln_quant_kernel<W, VPT>, threads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int need = (T + RPB - 1) / RPB;
  int grid = num_sms() * per_sm;
  if (grid > need) grid = need;
  const double c1 = 0x1p-24 / static_cast<double>(K);
  const double c2 = 0x1p-48 / static_cast<double>(K);
  e = launch_pdl(ln_quant_kernel<W, VPT>, dim3(grid), dim3(threads), 0, st, X, g, b, T, K, eps,
                 c1, c2, Xq, s, Y);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int W>
cudaError_t launch_ln_w(int vpt, const __half* X, const __half* g, const __half* b, int T, int K,
                        float eps, int8_t* Xq, float* s, __half* Y, cudaStream_t st) {
  switch (vpt) {
    case 1: return launch_ln<W, 1>(X, g, b, T, K, eps, Xq, s, Y, st);
    case 2: return launch_ln<W, 2>(X, g, b, T, K, eps, Xq, s, Y, st);
    case 3: return launch_ln<W, 3>(X, g, b, T, K, eps, Xq, s, Y, st);
    default: return launch_ln<W, 4>(X, g, b, T, K, eps, Xq, s, Y, st);
  }
}

// ----------------------------------------------------------------- wquant

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x / 32, nw = blockDim.x / 32;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = 0.0f;
  for (int i = 0; i < nw; ++i) m = fmaxf(m, red[i]);
  return m;
}

// One CTA per group i: rows o with floor(o*g/N) == i, i.e. o in
// [ceil(i*N/g), ceil((i+1)*N/g)).  Pass 1: group absmax; pass 2: codes.
__global__ void __launch_bounds__(512) wquant_kernel(const __half* __restrict__ W, int N, int K,
                                                     int g, int bits, void* __restrict__ Wq,
                                                     float* __restrict__ s_grp) {
  __shared__ float red[16];
  grid_dependency_wait();
  grid_launch_dependents();
  const int i = blockIdx.x;
  const long long r0 = (static_cast<long long>(i) * N + g - 1) / g;
  const long long r1 = (static_cast<long long>(i + 1) * N + g - 1) / g;
  const long long nv = (r1 - r0) * (K / 8);  // 8-half vectors in the group
  const uint4* src = reinterpret_cast<const uint4*>(W + r0 * K);
  const float qmax = bits == 8 ? 127.0f : 7.0f;

  float amax = 0.0f;
  for (long long v = threadIdx.x; v < nv; v += blockDim.x) {
    uint4 x = __ldg(src + v);
    const __half* h = reinterpret_cast<const __half*>(&x);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(__half2float(h[e])));
  }
  amax = block_max(amax, red);
  const float inv = amax > 0.0f ? __fdiv_rn(qmax, amax) : 0.0f;
  if (threadIdx.x == 0) s_grp[i] = amax > 0.0f ? __fdiv_rn(amax, qmax) : 0.0f;

  for (long long v = threadIdx.x; v < nv; v += blockDim.x) {
    uint4 x = __ldg(src + v);
    const __half* h = reinterpret_cast<const __half*>(&x);
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = quant_code(__half2float(h[e]), inv, qmax);
    if (bits == 8) {
      uint2 out;
      out.x = pack4(c[0], c[1], c[2], c[3]);
      out.y = pack4(c[4], c[5], c[6], c[7]);
      reinterpret_cast<uint2*>(static_cast<int8_t*>(Wq) + r0 * K)[v] = out;
    } else {
      // two's-complement nibbles; of eight consecutive k, byte i holds
      // k = i (low nibble) and k = 4 + i (high nibble)
      uint32_t out = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) out |= ((c[e] & 0xFu) | ((c[e + 4] & 0xFu) << 4)) << (8 * e);
      reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(Wq) + r0 * (K / 2))[v] = out;
    }
  }
}

}  // namespace
}  // namespace zq

using namespace zq;

extern "C" zq_status zq_ln_quant(const void* X, const void* gamma, const void* beta, int T, int K,
                                 float eps, int8_t* Xq, float* s_tok, void* Y_ln,
                                 zq_stream_t stream) {
  if (T < 0 || K < 16 || K > 32768 || K % 16 != 0) return ZQ_ERR_SHAPE;
  if (T == 0) return ZQ_OK;
  if (!X || !Xq || !s_tok) return ZQ_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || (gamma && !aligned16(gamma)) ||
      (gamma && beta && !aligned16(beta)) || (Y_ln && !aligned16(Y_ln)))
    return ZQ_ERR_ALIGN;
  const __half* xg = static_cast<const __half*>(X);
  const __half* gg = static_cast<const __half*>(gamma);
  const __half* bg = gamma ? static_cast<const __half*>(beta) : nullptr;
  __half* yg = static_cast<__half*>(Y_ln);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // warps per row so that each thread keeps at most 4 vectors of 8 halves
  const int nvec = K / 8;
  int W = 1;
  while (W < 32 && 32 * W * 4 < nvec) W *= 2;
  const int vpt = (nvec + 32 * W - 1) / (32 * W);
  cudaError_t e;
  switch (W) {
    case 1: e = launch_ln_w<1>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st); break;
    case 2: e = launch_ln_w<2>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st); break;
    case 4: e = launch_ln_w<4>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st); break;
    case 8: e = launch_ln_w<8>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st); break;
    case 16: e = launch_ln_w<16>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st); break;
    default: e = launch_ln_w<32>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st); break;
  }
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

extern "C" zq_status zq_quantize_weights_groupwise(const void* W, int N, int K, int g, int bits,
                                                   void* Wq, float* s_grp, zq_stream_t stream) {
  if (bits != 8 && bits != 4) return ZQ_ERR_UNSUPPORTED;
  if (N < 1 || K < 16 || K % 16 != 0 || g < 1 || g > N) return ZQ_ERR_SHAPE;
  if (bits == 4 && K % 32 != 0) return ZQ_ERR_SHAPE;
  if (!W || !Wq || !s_grp) return ZQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(Wq)) return ZQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (launch_pdl(wquant_kernel, dim3(g), dim3(512), 0, st, static_cast<const __half*>(W), N, K, g,
                 bits, Wq, s_grp) != cudaSuccess)
    return ZQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}
