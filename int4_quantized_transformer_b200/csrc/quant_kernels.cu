// quant_kernels.cu -- the two HBM-bound quantizers of the fused quantized
// linear layer (ZeroQuant, arXiv 2206.01861, Sec. 3.4):
//
//  * ln_quant: fused LayerNorm + token-wise dynamic INT8 quantization
//    ("Kernel fusion for token-wise activation quantization", Fig. 2 right):
//    each row is read once into registers with 128-bit loads; its mean and
//    variance (fp32 sums in a fixed chunk-and-tree order, two passes over
//    the registers), fp16 LayerNorm output and absmax are reduced with warp
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

// erfc(a) for a >= 0 in fp32: the Chebyshev approximation of Press, Teukolsky,
// Vetterling and Flannery, "Numerical Recipes", Sec. 6.2 (erfc with
// fractional error below 1.2e-7 everywhere), as
//   erfc(a) ~ t * exp(-a^2 + P(t)),  t = 1 / (1 + a/2),
// P a degree-9 polynomial, with the hardware exp2.  Fractional (not absolute)
// accuracy matters here: for negative v, GeLU is v times a tiny erfc.
__device__ __forceinline__ float erfc_nonneg(float a) {
  const float t = __frcp_rn(__fmaf_rn(0.5f, a, 1.0f));
  float p = 0.17087277f;
  p = __fmaf_rn(p, t, -0.82215223f);
  p = __fmaf_rn(p, t, 1.48851587f);
  p = __fmaf_rn(p, t, -1.13520398f);
  p = __fmaf_rn(p, t, 0.27886807f);
  p = __fmaf_rn(p, t, -0.18628806f);
  p = __fmaf_rn(p, t, 0.09678418f);
  p = __fmaf_rn(p, t, 0.37409196f);
  p = __fmaf_rn(p, t, 1.00002368f);
  p = __fmaf_rn(p, t, -1.26551223f);
  return t * __expf(__fmaf_rn(-a, a, p));
}

// GeLU, exact form: v * Phi(v) with Phi(v) = 0.5 erfc(-v / sqrt 2), i.e.
// 0.5 erfc(|v|/sqrt 2) for v <= 0 and 1 - 0.5 erfc(v/sqrt 2) for v > 0 (no
// cancellation for negative v).  The result stays well within an fp16 ulp of
// the correctly rounded value; the tests hold it to one fp16 ulp.
__device__ __forceinline__ float gelu_erf(float v) {
  const float h = 0.5f * erfc_nonneg(fabsf(v) * 0.70710678118654752f);
  return v * (v > 0.0f ? 1.0f - h : h);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Row sums in a fixed order that does not depend on the launch shape.  The
// row is cut into chunks of eight consecutive elements, each summed in
// order; the chunk sums, padded with zeros to a power of two, are combined
// by a pairwise tree (level l adds chunk c + 2^l into chunk c, for c a
// multiple of 2^(l+1)).  Chunk c sits in thread (c mod RT) of the row, slot
// c / RT, i.e. lane c mod 32 and "block" b = c / 32 = warp + W*slot, so
// levels 0..4 are xor-shuffles inside a warp (IEEE addition is commutative,
// so both partners hold the same bits) and the higher levels are the same
// tree over the blocks b.  `cs` holds this thread's chunk sums; the result
// reaches every thread of the row.
template <int W, int VPT>
__device__ __forceinline__ float row_tree_sum(float (&cs)[VPT], float* red, int lane, int wrow) {
  constexpr int VPTP = VPT <= 1 ? 1 : (VPT <= 2 ? 2 : 4);  // slots padded to a power of two
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < VPT; ++i) cs[i] = __fadd_rn(cs[i], __shfl_xor_sync(0xffffffffu, cs[i], o));
  if (W == 1) {  // blocks are the slots of this thread
    float b[VPTP];
#pragma unroll
    for (int i = 0; i < VPTP; ++i) b[i] = i < VPT ? cs[i] : 0.0f;
#pragma unroll
    for (int st = 1; st < VPTP; st <<= 1)
#pragma unroll
      for (int i = 0; i < VPTP; i += 2 * st) b[i] = __fadd_rn(b[i], b[i + st]);
    return b[0];
  }
  // W > 1: block b = warp + W*slot; every warp reduces all blocks from
  // shared memory (lane + 32r = b), first across lanes, then across r.
  constexpr int NB = W * VPTP;
  constexpr int NR = NB <= 32 ? 1 : NB / 32;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < VPTP; ++i) red[wrow + W * i] = i < VPT ? cs[i] : 0.0f;
  }
  __syncthreads();
  float v[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) v[r] = (lane + 32 * r < NB) ? red[lane + 32 * r] : 0.0f;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int r = 0; r < NR; ++r) v[r] = __fadd_rn(v[r], __shfl_xor_sync(0xffffffffu, v[r], o));
#pragma unroll
  for (int st = 1; st < NR; st <<= 1)
#pragma unroll
    for (int r = 0; r < NR; r += 2 * st) v[r] = __fadd_rn(v[r], v[r + st]);
  return v[0];
}

// Packed fp32 arithmetic of sm_100 (PTX ISA 8.6): two independent IEEE
// round-to-nearest operations per instruction (f32x2).  They give the same
// bits as the scalar operations, with fewer instructions per element.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
// running max of |.| over packed fp16 pairs (the sign of the result is
// meaningless; its magnitude is max(|a|, |b|) per half)
__device__ __forceinline__ uint32_t hmax_abs2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float habs_max(uint32_t m2) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&m2));
  return fmaxf(fabsf(f.x), fabsf(f.y));
}

// L2 prefetch of one fp16 row of K values (K % 8 == 0, 16-byte aligned),
// in bulk requests of at most 64 KB.
__device__ __forceinline__ void prefetch_row_l2(const __half* v, int K) {
  const char* p = reinterpret_cast<const char*>(v);
  for (uint32_t left = static_cast<uint32_t>(K) * 2u; left > 0;) {
    const uint32_t n = left < 65536u ? left : 65536u;
    bulk_prefetch_l2(p, n);
    p += n;
    left -= n;
  }
}

// ------------------------------------------------- token quantization only

// One row per group of W warps, VPT 16-byte vectors (8 halves) per thread:
// the quant-only form of zq_ln_quant, zq_bias_act_quant (act >= 0: the
// bias-add or GeLU producer fused in front) and zq_static_quant
// (static_amax >= 0).  Blocks hold RPB = max(1, 8/W) rows; every thread
// runs the same number of row iterations so block-wide barriers stay
// uniform.  The loads of a thread's next row are issued before the current
// row is reduced, so their latency overlaps its arithmetic.
template <int W, int VPT>
__global__ void __launch_bounds__((W >= 8 ? W : 8) * 32, (W >= 8 ? 2048 / (W * 32) : 8) / 2)
    quant_rows_kernel(const __half* __restrict__ X, const __half* __restrict__ act_bias, int act,
                      float static_amax, int T, int K, int8_t* __restrict__ Xq,
                      float* __restrict__ s_tok, __half* __restrict__ Y_out) {
  constexpr int RT = 32 * W;                // threads per row
  constexpr int RPB = W >= 8 ? 1 : 8 / W;   // rows per block
  __shared__ float red_m[RPB][W];

  const int slot = threadIdx.x / RT;
  const int j = threadIdx.x % RT;
  const int warp_in_row = j / 32;
  const int lane = threadIdx.x & 31;
  const int nvec = K / 8;
  // the bias of the bias-add / GeLU form, as gamma and beta in ln_rows2_kernel
  if (act_bias && blockIdx.x == 0 && threadIdx.x == 0) prefetch_row_l2(act_bias, K);
  grid_dependency_wait();
  grid_launch_dependents();

  const int rows_per_iter = gridDim.x * RPB;
  const int iters = (T + rows_per_iter - 1) / rows_per_iter;
  auto load_row = [&](uint4 (&dst)[VPT], int row) {
    const __half* xr = X + static_cast<size_t>(row) * K;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = j + i * RT;
      dst[i] = make_uint4(0, 0, 0, 0);
      if (row < T && v < nvec) dst[i] = __ldcs(reinterpret_cast<const uint4*>(xr) + v);
    }
  };
  uint4 x4[VPT];
  load_row(x4, blockIdx.x * RPB + slot);
  for (int it = 0; it < iters; ++it) {
    const int row = (it * gridDim.x + blockIdx.x) * RPB + slot;
    const bool valid = row < T;
    uint4 n4[VPT];
    if (it + 1 < iters) load_row(n4, ((it + 1) * gridDim.x + blockIdx.x) * RPB + slot);

    if (act >= 0) {
      // the producer of the activation, fused: bias-add (act = 0) or
      // GeLU (act = 1) of v = f32(x) + f32(bias), rounded to fp16 (the
      // bias-add is skipped when there is no bias, so x stays bit-exact)
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int v = j + i * RT;
        if (v < nvec) {
          const uint4 b4 = act_bias ? __ldg(reinterpret_cast<const uint4*>(act_bias) + v)
                                    : make_uint4(0, 0, 0, 0);
          __half2* h = reinterpret_cast<__half2*>(&x4[i]);
          const __half2* bh = reinterpret_cast<const __half2*>(&b4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float2 f = __half22float2(h[e]);
            if (act_bias) {
              const float2 bf = __half22float2(bh[e]);
              f.x = __fadd_rn(f.x, bf.x);
              f.y = __fadd_rn(f.y, bf.y);
            }
            if (act == 1) {
              f.x = gelu_erf(f.x);
              f.y = gelu_erf(f.y);
            }
            h[e] = __floats2half2_rn(f.x, f.y);
          }
        }
      }
    }

    // static quantization: one calibrated range for every token (codes may
    // then exceed the range and are clamped), no per-row reduction
    const bool is_static = static_amax >= 0.0f;  // uniform over the grid
    float amax = static_amax;
    if (!is_static) {
      uint32_t m2 = 0u;  // padding vectors are zero
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&x4[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) m2 = hmax_abs2(m2, w[e]);
      }
      amax = warp_max(habs_max(m2));
      if (W > 1) {
        if (lane == 0) red_m[slot][warp_in_row] = amax;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < W; ++w) amax = fmaxf(amax, red_m[slot][w]);
        __syncthreads();  // red_m is reused by the next row
      }
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
            c[2 * e] = is_static ? quant_code(f.x, inv, 127.0f) : token_code(f.x, inv);
            c[2 * e + 1] = is_static ? quant_code(f.y, inv, 127.0f) : token_code(f.y, inv);
          }
          uint2 out;
          out.x = pack4(c[0], c[1], c[2], c[3]);
          out.y = pack4(c[4], c[5], c[6], c[7]);
          __stcs(reinterpret_cast<uint2*>(qr) + v, out);
          if (Y_out) reinterpret_cast<uint4*>(Y_out + static_cast<size_t>(row) * K)[v] = x4[i];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) x4[i] = n4[i];
  }
}

// ---------------------------------------------------------- LN + quant

// The fixed-order tree of row_tree_sum for two rows at once: the low and
// high halves of each f32x2 value are rows A and B, and every add is the
// same IEEE operation as in the one-row tree.
template <int W, int VPT>
__device__ __forceinline__ uint64_t row_tree_sum2(uint64_t (&cs)[VPT], uint64_t* red, int lane,
                                                  int wrow) {
  constexpr int VPTP = VPT <= 1 ? 1 : (VPT <= 2 ? 2 : 4);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < VPT; ++i) cs[i] = f2_add(cs[i], __shfl_xor_sync(0xffffffffu, cs[i], o));
  if (W == 1) {
    uint64_t b[VPTP];
#pragma unroll
    for (int i = 0; i < VPTP; ++i) b[i] = i < VPT ? cs[i] : 0ull;
#pragma unroll
    for (int st = 1; st < VPTP; st <<= 1)
#pragma unroll
      for (int i = 0; i < VPTP; i += 2 * st) b[i] = f2_add(b[i], b[i + st]);
    return b[0];
  }
  constexpr int NB = W * VPTP;
  constexpr int NR = NB <= 32 ? 1 : NB / 32;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < VPTP; ++i) red[wrow + W * i] = i < VPT ? cs[i] : 0ull;
  }
  __syncthreads();
  uint64_t v[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) v[r] = (lane + 32 * r < NB) ? red[lane + 32 * r] : 0ull;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int r = 0; r < NR; ++r) v[r] = f2_add(v[r], __shfl_xor_sync(0xffffffffu, v[r], o));
#pragma unroll
  for (int st = 1; st < NR; st <<= 1)
#pragma unroll
    for (int r = 0; r < NR; r += 2 * st) v[r] = f2_add(v[r], v[r + st]);
  return v[0];
}

// Fused LayerNorm + token quantization, two rows (A = 2p, B = 2p + 1) per
// group of W warps.  Each thread holds VPT 16-byte vectors of both rows and
// keeps every per-column value as an f32x2 pair (row A, row B), so the
// statistics, the deviations and the quantization run two rows per
// instruction with the one-row operation order: chunk sums in index order,
// the fixed tree, the two-pass variance with fused multiply-adds, then
// y = fp16(((x - mean) * rstd) * gamma + beta) with each step rounded once.
// Blocks hold PPB = max(1, 8/W) row pairs; the next pair's loads are issued
// before the current pair is reduced.
template <int W, int VPT>
__global__ void __launch_bounds__((W >= 8 ? W : 8) * 32)
    ln_rows2_kernel(const __half* __restrict__ X, const __half* __restrict__ gamma,
                    const __half* __restrict__ beta, int T, int K, float eps,
                    int8_t* __restrict__ Xq, float* __restrict__ s_tok,
                    __half* __restrict__ Y_ln) {
  constexpr int RT = 32 * W;                // threads per row pair
  constexpr int PPB = W >= 8 ? 1 : 8 / W;   // row pairs per block
  constexpr int NBLK = W * (VPT <= 1 ? 1 : (VPT <= 2 ? 2 : 4));
  __shared__ uint64_t red1[PPB][NBLK];  // block sums of x (W > 1)
  __shared__ uint64_t red2[PPB][NBLK];  // block sums of (x - mean)^2 (W > 1)
  __shared__ float red_m[PPB][2][W];

  const int slot = threadIdx.x / RT;
  const int j = threadIdx.x % RT;
  const int warp_in_row = j / 32;
  const int lane = threadIdx.x & 31;
  const int nvec = K / 8;
  // gamma and beta are read only after the row statistics: ask L2 for them
  // now, before waiting for the previous kernel of the stream, so that their
  // DRAM latency overlaps the wait and the reductions (an L2 prefetch, which
  // every kernel's writes reach coherently, so a stale read is impossible).
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    prefetch_row_l2(gamma, K);
    if (beta) prefetch_row_l2(beta, K);
  }
  grid_dependency_wait();
  grid_launch_dependents();

  const int pairs = (T + 1) / 2;
  const int pairs_per_iter = gridDim.x * PPB;
  const int iters = (pairs + pairs_per_iter - 1) / pairs_per_iter;
  auto load_pair = [&](uint4 (&a)[VPT], uint4 (&b)[VPT], int p) {
    const __half* xa = X + static_cast<size_t>(2 * p) * K;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = j + i * RT;
      a[i] = make_uint4(0, 0, 0, 0);
      b[i] = make_uint4(0, 0, 0, 0);
      if (v < nvec) {
        if (2 * p < T) a[i] = __ldcs(reinterpret_cast<const uint4*>(xa) + v);
        if (2 * p + 1 < T) b[i] = __ldcs(reinterpret_cast<const uint4*>(xa + K) + v);
      }
    }
  };
  uint4 xa[VPT], xb[VPT];
  load_pair(xa, xb, blockIdx.x * PPB + slot);
  for (int it = 0; it < iters; ++it) {
    const int p = (it * gridDim.x + blockIdx.x) * PPB + slot;
    uint4 na[VPT], nb[VPT];
    if (it + 1 < iters) load_pair(na, nb, ((it + 1) * gridDim.x + blockIdx.x) * PPB + slot);

    // x as (row A, row B) pairs; chunk sums in index order
    uint64_t P[VPT][8];
    uint64_t cs[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const __half* ha = reinterpret_cast<const __half*>(&xa[i]);
      const __half* hb = reinterpret_cast<const __half*>(&xb[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) P[i][e] = f2_pack(__half2float(ha[e]), __half2float(hb[e]));
      uint64_t acc = f2_add(P[i][0], P[i][1]);
#pragma unroll
      for (int e = 2; e < 8; ++e) acc = f2_add(acc, P[i][e]);
      cs[i] = acc;  // zero for chunks past the row (the vectors are zero there)
    }
    float sa, sb;
    f2_unpack(row_tree_sum2<W, VPT>(cs, red1[slot], lane, warp_in_row), sa, sb);
    const float mean_a = __fdiv_rn(sa, static_cast<float>(K));
    const float mean_b = __fdiv_rn(sb, static_cast<float>(K));
    // deviations x - mean (as x + (-mean), the same IEEE operation), then the
    // biased variance: per chunk the first square, then fused multiply-adds
    const uint64_t negm = f2_pack(-mean_a, -mean_b);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
#pragma unroll
      for (int e = 0; e < 8; ++e) P[i][e] = f2_add(P[i][e], negm);
      uint64_t q = f2_mul(P[i][0], P[i][0]);
#pragma unroll
      for (int e = 1; e < 8; ++e) q = f2_fma(P[i][e], P[i][e], q);
      cs[i] = (j + i * RT < nvec) ? q : 0ull;  // padding chunks are zero
    }
    f2_unpack(row_tree_sum2<W, VPT>(cs, red2[slot], lane, warp_in_row), sa, sb);
    const float var_a = __fdiv_rn(sa, static_cast<float>(K));
    const float var_b = __fdiv_rn(sb, static_cast<float>(K));
    const uint64_t rstd2 = f2_pack(__fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var_a, eps))),
                                   __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var_b, eps))));
    // y = fp16(((x - mean) * rstd) * gamma + beta): the first product for
    // both rows at once, gamma and beta (shared by the rows) one row at a time
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = j + i * RT;
      if (v < nvec) {
        const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
        const uint4 b4 = beta ? __ldg(reinterpret_cast<const uint4*>(beta) + v)
                              : make_uint4(0, 0, 0, 0);
        const __half2* gh = reinterpret_cast<const __half2*>(&g4);
        const __half2* bh = reinterpret_cast<const __half2*>(&b4);
        __half2* ya = reinterpret_cast<__half2*>(&xa[i]);
        __half2* yb = reinterpret_cast<__half2*>(&xb[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 gf = __half22float2(gh[e]);
          const float2 bf = __half22float2(bh[e]);
          float a0, b0, a1, b1;
          f2_unpack(f2_mul(P[i][2 * e], rstd2), a0, b0);
          f2_unpack(f2_mul(P[i][2 * e + 1], rstd2), a1, b1);
          ya[e] = __floats2half2_rn(__fadd_rn(__fmul_rn(a0, gf.x), bf.x),
                                    __fadd_rn(__fmul_rn(a1, gf.y), bf.y));
          yb[e] = __floats2half2_rn(__fadd_rn(__fmul_rn(b0, gf.x), bf.x),
                                    __fadd_rn(__fmul_rn(b1, gf.y), bf.y));
        }
      } else {
        xa[i] = make_uint4(0, 0, 0, 0);
        xb[i] = make_uint4(0, 0, 0, 0);
      }
    }
    // absmax of both fp16 rows
    uint32_t ma = 0u, mb = 0u;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const uint32_t* wa = reinterpret_cast<const uint32_t*>(&xa[i]);
      const uint32_t* wb = reinterpret_cast<const uint32_t*>(&xb[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ma = hmax_abs2(ma, wa[e]);
        mb = hmax_abs2(mb, wb[e]);
      }
    }
    float amax_a = warp_max(habs_max(ma));
    float amax_b = warp_max(habs_max(mb));
    if (W > 1) {
      if (lane == 0) {
        red_m[slot][0][warp_in_row] = amax_a;
        red_m[slot][1][warp_in_row] = amax_b;
      }
      __syncthreads();
#pragma unroll
      for (int w = 0; w < W; ++w) {
        amax_a = fmaxf(amax_a, red_m[slot][0][w]);
        amax_b = fmaxf(amax_b, red_m[slot][1][w]);
      }
      __syncthreads();  // red1 / red2 / red_m are reused by the next pair
    }
    const float inv_a = amax_a > 0.0f ? __fdiv_rn(127.0f, amax_a) : 0.0f;
    const float inv_b = amax_b > 0.0f ? __fdiv_rn(127.0f, amax_b) : 0.0f;
    const int ra = 2 * p, rb = 2 * p + 1;
    if (j == 0) {
      if (ra < T) s_tok[ra] = amax_a > 0.0f ? __fdiv_rn(amax_a, 127.0f) : 0.0f;
      if (rb < T) s_tok[rb] = amax_b > 0.0f ? __fdiv_rn(amax_b, 127.0f) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = j + i * RT;
      if (v < nvec) {
        const __half2* ya = reinterpret_cast<const __half2*>(&xa[i]);
        const __half2* yb = reinterpret_cast<const __half2*>(&xb[i]);
        uint32_t ca[8], cb[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = __half22float2(ya[e]);
          const float2 fb = __half22float2(yb[e]);
          ca[2 * e] = token_code(fa.x, inv_a);
          ca[2 * e + 1] = token_code(fa.y, inv_a);
          cb[2 * e] = token_code(fb.x, inv_b);
          cb[2 * e + 1] = token_code(fb.y, inv_b);
        }
        if (ra < T) {
          __stcs(reinterpret_cast<uint2*>(Xq + static_cast<size_t>(ra) * K) + v,
                 make_uint2(pack4(ca[0], ca[1], ca[2], ca[3]), pack4(ca[4], ca[5], ca[6], ca[7])));
          if (Y_ln) reinterpret_cast<uint4*>(Y_ln + static_cast<size_t>(ra) * K)[v] = xa[i];
        }
        if (rb < T) {
          __stcs(reinterpret_cast<uint2*>(Xq + static_cast<size_t>(rb) * K) + v,
                 make_uint2(pack4(cb[0], cb[1], cb[2], cb[3]), pack4(cb[4], cb[5], cb[6], cb[7])));
          if (Y_ln) reinterpret_cast<uint4*>(Y_ln + static_cast<size_t>(rb) * K)[v] = xb[i];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      xa[i] = na[i];
      xb[i] = nb[i];
    }
  }
}

// Launches on as many CTAs as are resident at once, or fewer when there are
// fewer row groups (the row loop is grid-strided).
template <class Kern, class... Args>
cudaError_t launch_resident(Kern kernel, int threads, int groups, cudaStream_t st, Args... args) {
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int grid = num_sms() * per_sm;
  if (grid > groups) grid = groups;
  if (grid < 1) grid = 1;
  e = launch_pdl(kernel, dim3(grid), dim3(threads), 0, st, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int W, int VPT>
cudaError_t launch_quant_rows(const __half* X, const __half* ab, int act, float sa, int T, int K,
                              int8_t* Xq, float* s, __half* Y, cudaStream_t st) {
  constexpr int RPB = W >= 8 ? 1 : 8 / W;
  return launch_resident(quant_rows_kernel<W, VPT>, RPB * 32 * W, (T + RPB - 1) / RPB, st, X, ab,
                         act, sa, T, K, Xq, s, Y);
}

template <int W, int VPT>
cudaError_t launch_ln_rows2(const __half* X, const __half* g, const __half* b, int T, int K,
                            float eps, int8_t* Xq, float* s, __half* Y, cudaStream_t st) {
  constexpr int PPB = W >= 8 ? 1 : 8 / W;
  const int pairs = (T + 1) / 2;
  return launch_resident(ln_rows2_kernel<W, VPT>, PPB * 32 * W, (pairs + PPB - 1) / PPB, st, X, g,
                         b, T, K, eps, Xq, s, Y);
}

#define ZQ_VPT_SWITCH(FN, W, vpt, ...)                  \
  switch (vpt) {                                        \
    case 1: return FN<W, 1>(__VA_ARGS__);               \
    case 2: return FN<W, 2>(__VA_ARGS__);               \
    case 3: return FN<W, 3>(__VA_ARGS__);               \
    default: return FN<W, 4>(__VA_ARGS__);              \
  }

template <int W>
cudaError_t launch_quant_w(int vpt, const __half* X, const __half* ab, int act, float sa, int T,
                           int K, int8_t* Xq, float* s, __half* Y, cudaStream_t st) {
  ZQ_VPT_SWITCH(launch_quant_rows, W, vpt, X, ab, act, sa, T, K, Xq, s, Y, st)
}

template <int W>
cudaError_t launch_ln_w(int vpt, const __half* X, const __half* g, const __half* b, int T, int K,
                        float eps, int8_t* Xq, float* s, __half* Y, cudaStream_t st) {
  switch (vpt) {
    case 1: return launch_ln_rows2<W, 1>(X, g, b, T, K, eps, Xq, s, Y, st);
    case 2: return launch_ln_rows2<W, 2>(X, g, b, T, K, eps, Xq, s, Y, st);
    default: return launch_ln_rows2<W, 3>(X, g, b, T, K, eps, Xq, s, Y, st);
  }
}

// Warps per row so that each thread keeps at most 4 vectors of 8 halves
// (3 for the two-row LayerNorm kernel, which holds both rows); act < 0
// selects the LayerNorm (gamma non-NULL) or quant-only form; sa >= 0 is a
// static range (one scale for every token).
cudaError_t launch_row_quant(const __half* xg, const __half* gg, const __half* bg,
                             const __half* ab, int act, float sa, int T, int K, float eps,
                             int8_t* Xq, float* s_tok, __half* yg, cudaStream_t st) {
  const int nvec = K / 8;
  const int vmax = gg ? 3 : 4;
  int W = 1;
  while (W < 32 && 32 * W * vmax < nvec) W *= 2;
  const int vpt = (nvec + 32 * W - 1) / (32 * W);
  if (gg) {
    switch (W) {
      case 1: return launch_ln_w<1>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st);
      case 2: return launch_ln_w<2>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st);
      case 4: return launch_ln_w<4>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st);
      case 8: return launch_ln_w<8>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st);
      case 16: return launch_ln_w<16>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st);
      default: return launch_ln_w<32>(vpt, xg, gg, bg, T, K, eps, Xq, s_tok, yg, st);
    }
  }
  switch (W) {
    case 1: return launch_quant_w<1>(vpt, xg, ab, act, sa, T, K, Xq, s_tok, yg, st);
    case 2: return launch_quant_w<2>(vpt, xg, ab, act, sa, T, K, Xq, s_tok, yg, st);
    case 4: return launch_quant_w<4>(vpt, xg, ab, act, sa, T, K, Xq, s_tok, yg, st);
    case 8: return launch_quant_w<8>(vpt, xg, ab, act, sa, T, K, Xq, s_tok, yg, st);
    case 16: return launch_quant_w<16>(vpt, xg, ab, act, sa, T, K, Xq, s_tok, yg, st);
    default: return launch_quant_w<32>(vpt, xg, ab, act, sa, T, K, Xq, s_tok, yg, st);
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
  const cudaError_t e =
      launch_row_quant(xg, gg, bg, nullptr, -1, -1.0f, T, K, eps, Xq, s_tok, yg, st);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

extern "C" zq_status zq_bias_act_quant(const void* X, const void* bias, int T, int K, int act,
                                       int8_t* Xq, float* s_tok, void* Y_act,
                                       zq_stream_t stream) {
  if (act != ZQ_ACT_NONE && act != ZQ_ACT_GELU) return ZQ_ERR_UNSUPPORTED;
  if (T < 0 || K < 16 || K > 32768 || K % 16 != 0) return ZQ_ERR_SHAPE;
  if (T == 0) return ZQ_OK;
  if (!X || !Xq || !s_tok) return ZQ_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || (bias && !aligned16(bias)) ||
      (Y_act && !aligned16(Y_act)))
    return ZQ_ERR_ALIGN;
  const cudaError_t e = launch_row_quant(
      static_cast<const __half*>(X), nullptr, nullptr, static_cast<const __half*>(bias), act, -1.0f,
      T, K, 0.0f, Xq, s_tok, static_cast<__half*>(Y_act), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

extern "C" zq_status zq_static_quant(const void* X, int T, int K, float amax, int8_t* Xq,
                                     float* s_tok, zq_stream_t stream) {
  if (!(amax >= 0.0f) || amax > 65504.0f) return ZQ_ERR_SHAPE;  // also rejects NaN
  if (T < 0 || K < 16 || K > 32768 || K % 16 != 0) return ZQ_ERR_SHAPE;
  if (T == 0) return ZQ_OK;
  if (!X || !Xq || !s_tok) return ZQ_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq)) return ZQ_ERR_ALIGN;
  const cudaError_t e = launch_row_quant(static_cast<const __half*>(X), nullptr, nullptr, nullptr,
                                         -1, amax, T, K, 0.0f, Xq, s_tok, nullptr,
                                         reinterpret_cast<cudaStream_t>(stream));
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
