// zq_internal.h -- declarations shared by the translation units of libzq.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "zq.h"

namespace zq {

// Bounded device-side waits give up after this long (about one second).
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;
// Device status word values: 0 = fine; kDevErrTimeoutBase + site = a wait
// at `site` gave up.
constexpr int kDevErrTimeoutBase = 1000;

// Device pointer of the current device's status word (set up once per device).
int* device_status_ptr();
int num_sms();

// The CUDA-core matrix-vector path of the quantized linear layer, for at most
// kGemvMaxTokens tokens (gemv_i8.cu): bits = 4 (packed INT4) or 8.
constexpr int kGemvMaxTokens = 4;
cudaError_t launch_gemv_i8(int bits, const int8_t* Xq, const float* s_tok, const void* W,
                           const float* s_grp, int g, const void* bias, int T, int N, int K,
                           void* Y, int32_t* acc_dbg, int max_ctas, cudaStream_t st);
// The CUDA-core matrix-vector path of the FP16-activation layer (gemv_a16.cu),
// for at most kGemvA16MaxTokens tokens: bits = 4 (packed INT4) or 8.
constexpr int kGemvA16MaxTokens = 4;
cudaError_t launch_gemv_a16(int bits, const void* X, const void* W, const float* s_grp, int g,
                            const void* bias, int T, int N, int K, void* Y, float* acc_dbg,
                            int max_ctas, cudaStream_t st);
int option(int key);
// The library workspace of the current device (gemm_i8.cu): at least
// `bytes` bytes, grown with cudaMalloc when a call needs more than it holds
// (ZQ_ERR_UNSUPPORTED instead while `st` is being captured into a graph).
// One buffer per device; calls that use it on different streams must not
// overlap.
zq_status library_workspace(size_t bytes, cudaStream_t st, void** out);
// Counts one kernel launch issued by the library (zq_launch_count).
void count_launch();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
// Returns false when the driver entry point is unavailable or encoding fails.
bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                   uint32_t box_outer, CUtensorMapSwizzle swizzle);

// A 3-D tiled map over row-major [outer][inner] bytes viewed as
// [inner / slice][outer][slice]: one box fetches `box_slices` consecutive
// slices of `box_outer` rows (slice-major in shared memory).  `inner` must
// be a multiple of `slice`.
bool encode_tma_3d_slices(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                          uint32_t slice, uint32_t box_outer, uint32_t box_slices,
                          CUtensorMapSwizzle swizzle);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launches a kernel on `st` with programmatic stream serialization, so that
// it may be scheduled while the previous kernel of the stream finishes.
// Every libzq kernel calls grid_dependency_wait() before it touches global
// memory, so the stream order of reads and writes is unchanged.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// As launch_pdl, with thread-block clusters of `cluster_x` CTAs (cluster_x
// > 1; the grid must be a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace zq

#define ZQ_CUDA_OK(expr)                       \
  do {                                         \
    if ((expr) != cudaSuccess) return ZQ_ERR_CUDA; \
  } while (0)
