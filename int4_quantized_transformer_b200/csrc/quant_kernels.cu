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

#include <atomic>

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

// Packed and mixed-precision fp32 arithmetic of sm_100 (PTX ISA 8.6): two
// independent IEEE round-to-nearest operations per instruction (f32x2), and
// an add or subtract whose first operand is fp16 (converted exactly, then
// one rounding).  They give the same bits as the scalar operations, with
// fewer instructions per element.
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
// f32(h) + c and f32(h) - c, one rounding each
__device__ __forceinline__ float add_h(uint16_t h, float c) {
  float r;
  asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(r) : "h"(h), "f"(c));
  return r;
}
__device__ __forceinline__ float sub_h(uint16_t h, float c) {
  float r;
  asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(r) : "h"(h), "f"(c));
  return r;
}
__device__ __forceinline__ void halves(uint32_t w, uint16_t& lo, uint16_t& hi) {
  asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(w));
}
// running max of |.| over packed fp16 pairs (the sign of the result is
// meaningless; its magnitude is max(|a|, |b|) per half)
__device__ __forceinline__ uint32_t hmax_abs2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// LayerNorm gamma/beta are kept as fp32 in shared memory (converted once per
// CTA) when both fit in this many bytes; longer rows convert per row.
constexpr int kGammaBetaSmemMax = 64 * 1024;

// W warps per row, VPT 16-byte vectors (8 halves) per thread.  Blocks hold
// RPB = max(1, 8/W) rows; every thread runs the same number of row
// iterations so block-wide barriers stay uniform.  The loads of a thread's
// next row are issued before the current row is reduced, so their latency
// overlaps its arithmetic.
template <int W, int VPT>
__global__ void __launch_bounds__((W >= 8 ? W : 8) * 32)
    ln_quant_kernel(const __half* __restrict__ X, const __half* __restrict__ gamma,
                    const __half* __restrict__ beta, const __half* __restrict__ act_bias,
                    int act, float static_amax, int T, int K, float eps,
                    int8_t* __restrict__ Xq, float* __restrict__ s_tok,
                    __half* __restrict__ Y_ln) {
  constexpr int RT = 32 * W;                // threads per row
  constexpr int RPB = W >= 8 ? 1 : 8 / W;   // rows per block
  constexpr int NBLK = W * (VPT <= 1 ? 1 : (VPT <= 2 ? 2 : 4));
  __shared__ float red1[RPB][NBLK];  // block sums of x (W > 1)
  __shared__ float red2[RPB][NBLK];  // block sums of (x - mean)^2 (W > 1)
  __shared__ float red_m[RPB][W];
  extern __shared__ float4 gb_smem[];  // fp32 gamma [K], then beta [K] (when they fit)

  const int slot = threadIdx.x / RT;
  const int j = threadIdx.x % RT;
  const int warp_in_row = j / 32;
  const int lane = threadIdx.x & 31;
  const int nvec = K / 8;
  const bool ln = gamma != nullptr;
  const bool gb_smem_ok = ln && 8 * K <= kGammaBetaSmemMax;
  const float* g_s = reinterpret_cast<const float*>(gb_smem);
  const float* b_s = g_s + K;
  grid_dependency_wait();
  grid_launch_dependents();
  if (gb_smem_ok) {
    float* gs = reinterpret_cast<float*>(gb_smem);
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
      const uint4 b4 = beta ? __ldg(reinterpret_cast<const uint4*>(beta) + v) : make_uint4(0, 0, 0, 0);
      const __half2* gh = reinterpret_cast<const __half2*>(&g4);
      const __half2* bh = reinterpret_cast<const __half2*>(&b4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 gf = __half22float2(gh[e]);
        const float2 bf = __half22float2(bh[e]);
        gs[8 * v + 2 * e] = gf.x;
        gs[8 * v + 2 * e + 1] = gf.y;
        gs[K + 8 * v + 2 * e] = bf.x;
        gs[K + 8 * v + 2 * e + 1] = bf.y;
      }
    }
    __syncthreads();
  }

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

    if (ln) {
      // mean: each 8-element chunk summed in index order (the first element
      // plus -0 is the element itself, exactly), then the pairwise tree
      float cs[VPT];
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&x4[i]);
        float acc = -0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint16_t lo, hi;
          halves(w[e], lo, hi);
          acc = add_h(hi, add_h(lo, acc));
        }
        cs[i] = acc;  // zero for chunks past the row (x4 is zero there)
      }
      const float mean = __fdiv_rn(row_tree_sum<W, VPT>(cs, red1[slot], lane, warp_in_row),
                                   static_cast<float>(K));
      // deviations x - mean (kept for the normalisation), then the biased
      // variance: per chunk the first square, then fused multiply-adds in
      // index order, two chunks at a time in the two halves of f32x2
      float d[VPT][8];
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&x4[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint16_t lo, hi;
          halves(w[e], lo, hi);
          d[i][2 * e] = sub_h(lo, mean);
          d[i][2 * e + 1] = sub_h(hi, mean);
        }
      }
#pragma unroll
      for (int i = 0; i + 1 < VPT; i += 2) {
        uint64_t q = f2_pack(d[i][0], d[i + 1][0]);
        q = f2_mul(q, q);
#pragma unroll
        for (int e = 1; e < 8; ++e) {
          const uint64_t de = f2_pack(d[i][e], d[i + 1][e]);
          q = f2_fma(de, de, q);
        }
        f2_unpack(q, cs[i], cs[i + 1]);
      }
      if (VPT % 2) {
        float acc = __fmul_rn(d[VPT - 1][0], d[VPT - 1][0]);
#pragma unroll
        for (int e = 1; e < 8; ++e) acc = __fmaf_rn(d[VPT - 1][e], d[VPT - 1][e], acc);
        cs[VPT - 1] = acc;
      }
#pragma unroll
      for (int i = 0; i < VPT; ++i)
        if (j + i * RT >= nvec) cs[i] = 0.0f;  // padding chunks are zero
      const float var = __fdiv_rn(row_tree_sum<W, VPT>(cs, red2[slot], lane, warp_in_row),
                                  static_cast<float>(K));
      const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
      const uint64_t rstd2 = f2_pack(rstd, rstd);
      // y = fp16(((x - mean) * rstd) * gamma + beta), each step rounded once
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int v = j + i * RT;
        if (v < nvec) {
          float g[8], b[8];
          if (gb_smem_ok) {
            const float4* gp = reinterpret_cast<const float4*>(g_s + 8 * v);
            const float4* bp = reinterpret_cast<const float4*>(b_s + 8 * v);
            const float4 g0 = gp[0], g1 = gp[1], b0 = bp[0], b1 = bp[1];
            g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w;
            g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
            b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
            b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
          } else {
            const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(gamma) + v);
            const uint4 b4 = beta ? __ldg(reinterpret_cast<const uint4*>(beta) + v)
                                  : make_uint4(0, 0, 0, 0);
            const __half2* gh = reinterpret_cast<const __half2*>(&g4);
            const __half2* bh = reinterpret_cast<const __half2*>(&b4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 gf = __half22float2(gh[e]);
              const float2 bf = __half22float2(bh[e]);
              g[2 * e] = gf.x;
              g[2 * e + 1] = gf.y;
              b[2 * e] = bf.x;
              b[2 * e + 1] = bf.y;
            }
          }
          __half2* h = reinterpret_cast<__half2*>(&x4[i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint64_t t = f2_mul(f2_pack(d[i][2 * e], d[i][2 * e + 1]), rstd2);
            t = f2_mul(t, f2_pack(g[2 * e], g[2 * e + 1]));
            t = f2_add(t, f2_pack(b[2 * e], b[2 * e + 1]));
            float y0, y1;
            f2_unpack(t, y0, y1);
            h[e] = __floats2half2_rn(y0, y1);
          }
        }
      }
    }

    // absmax of the fp16 row (padding vectors are zero)
    uint32_t m2 = 0u;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&x4[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) m2 = hmax_abs2(m2, w[e]);
    }
    // static quantization: one calibrated range for every token (codes may
    // then exceed the range and are clamped), no per-row reduction
    const bool is_static = static_amax >= 0.0f;  // uniform over the grid
    float amax = static_amax;
    if (!is_static) {
      const float2 mf = __half22float2(*reinterpret_cast<const __half2*>(&m2));
      amax = warp_max(fmaxf(fabsf(mf.x), fabsf(mf.y)));
      if (W > 1) {
        if (lane == 0) red_m[slot][warp_in_row] = amax;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < W; ++w) amax = fmaxf(amax, red_m[slot][w]);
        __syncthreads();  // red1 / red2 / red_m are reused by the next row
      }
    }
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    const uint64_t inv2 = f2_pack(inv, inv);
    const uint64_t magic2 = f2_pack(12582912.0f, 12582912.0f);
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
            if (is_static) {
              c[2 * e] = quant_code(f.x, inv, 127.0f);
              c[2 * e + 1] = quant_code(f.y, inv, 127.0f);
            } else {
              // rne(y * inv) in the low byte: the product, then + 1.5 * 2^23
              const uint64_t t = f2_add(f2_mul(f2_pack(f.x, f.y), inv2), magic2);
              float a, b;
              f2_unpack(t, a, b);
              c[2 * e] = __float_as_uint(a);
              c[2 * e + 1] = __float_as_uint(b);
            }
          }
          uint2 out;
          out.x = pack4(c[0], c[1], c[2], c[3]);
          out.y = pack4(c[4], c[5], c[6], c[7]);
          __stcs(reinterpret_cast<uint2*>(qr) + v, out);
          if (Y_ln) reinterpret_cast<uint4*>(Y_ln + static_cast<size_t>(row) * K)[v] = x4[i];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) x4[i] = n4[i];
  }
}

template <int W, int VPT>
cudaError_t launch_ln(const __half* X, const __half* g, const __half* b, const __half* ab, int act,
                      float sa, int T, int K, float eps, int8_t* Xq, float* s, __half* Y,
                      cudaStream_t st) {
  constexpr int RPB = W >= 8 ? 1 : 8 / W;
  constexpr int threads = RPB * 32 * W;
  const size_t smem = (g && 8 * K <= kGammaBetaSmemMax) ? static_cast<size_t>(8) * K : 0;
  // per device; several host threads may race here, and a repeated set is
  // harmless
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(ln_quant_kernel<W, VPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGammaBetaSmemMax);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ln_quant_kernel<W, VPT>, threads,
                                                    smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int need = (T + RPB - 1) / RPB;
  int grid = num_sms() * per_sm;
  if (grid > need) grid = need;
  e = launch_pdl(ln_quant_kernel<W, VPT>, dim3(grid), dim3(threads), smem, st, X, g, b, ab, act,
                 sa, T, K, eps, Xq, s, Y);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int W>
cudaError_t launch_ln_w(int vpt, const __half* X, const __half* g, const __half* b,
                        const __half* ab, int act, float sa, int T, int K, float eps, int8_t* Xq,
                        float* s, __half* Y, cudaStream_t st) {
  switch (vpt) {
    case 1: return launch_ln<W, 1>(X, g, b, ab, act, sa, T, K, eps, Xq, s, Y, st);
    case 2: return launch_ln<W, 2>(X, g, b, ab, act, sa, T, K, eps, Xq, s, Y, st);
    case 3: return launch_ln<W, 3>(X, g, b, ab, act, sa, T, K, eps, Xq, s, Y, st);
    default: return launch_ln<W, 4>(X, g, b, ab, act, sa, T, K, eps, Xq, s, Y, st);
  }
}

// Warps per row so that each thread keeps at most 4 vectors of 8 halves;
// act < 0 selects the LayerNorm (gamma non-NULL) or quant-only form;
// sa >= 0 is a static range (one scale for every token).
cudaError_t launch_row_quant(const __half* xg, const __half* gg, const __half* bg,
                             const __half* ab, int act, float sa, int T, int K, float eps,
                             int8_t* Xq, float* s_tok, __half* yg, cudaStream_t st) {
  const int nvec = K / 8;
  int W = 1;
  while (W < 32 && 32 * W * 4 < nvec) W *= 2;
  const int vpt = (nvec + 32 * W - 1) / (32 * W);
  switch (W) {
    case 1: return launch_ln_w<1>(vpt, xg, gg, bg, ab, act, sa, T, K, eps, Xq, s_tok, yg, st);
    case 2: return launch_ln_w<2>(vpt, xg, gg, bg, ab, act, sa, T, K, eps, Xq, s_tok, yg, st);
    case 4: return launch_ln_w<4>(vpt, xg, gg, bg, ab, act, sa, T, K, eps, Xq, s_tok, yg, st);
    case 8: return launch_ln_w<8>(vpt, xg, gg, bg, ab, act, sa, T, K, eps, Xq, s_tok, yg, st);
    case 16: return launch_ln_w<16>(vpt, xg, gg, bg, ab, act, sa, T, K, eps, Xq, s_tok, yg, st);
    default: return launch_ln_w<32>(vpt, xg, gg, bg, ab, act, sa, T, K, eps, Xq, s_tok, yg, st);
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
