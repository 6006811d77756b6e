// zq_api.cu -- status codes, options, the per-device status word, TMA
// descriptor encoding and the bounded-wait self test of libzq.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "zq_internal.h"
#include "zq_ptx.cuh"

namespace zq {

// One status word per device (module-scope __device__ variable: no
// allocation).  Kernels write kDevErrTimeoutBase + site into it when a
// bounded wait gives up.
__device__ int g_dev_status;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
std::atomic<int> g_opts[8];
std::atomic<unsigned long long> g_launches{0};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}
}  // namespace

int* device_status_ptr() {
  int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_status) != cudaSuccess) return nullptr;
    g_status_ptr[d] = static_cast<int*>(p);
  }
  return g_status_ptr[d];
}

int num_sms() {
  int d = current_device();
  if (d < 0) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_num_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 148;
    g_num_sms[d] = n;
  }
  return g_num_sms[d];
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int option(int key) {
  if (key < 1 || key >= 8) return 0;
  return g_opts[key].load(std::memory_order_relaxed);
}

bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                   uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tma_3d_slices(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                          uint32_t slice, uint32_t box_outer, uint32_t box_slices,
                          CUtensorMapSwizzle swizzle) {
  if (slice == 0 || inner % slice != 0) return false;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t dims[3] = {slice, outer, inner / slice};
  cuuint64_t strides[2] = {inner, slice};  // bytes: next row, next slice
  cuuint32_t box[3] = {slice, box_outer, box_slices};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A barrier nobody arrives at: the wait must give up by itself.
__global__ void debug_wait_timeout_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, 1);
  __syncthreads();
}

}  // namespace zq

using namespace zq;

extern "C" {

const char* zq_status_str(int s) {
  switch (s) {
    case ZQ_OK: return "ZQ_OK";
    case ZQ_ERR_NULL: return "ZQ_ERR_NULL: a required pointer is NULL";
    case ZQ_ERR_SHAPE: return "ZQ_ERR_SHAPE: size out of range or inconsistent";
    case ZQ_ERR_ALIGN: return "ZQ_ERR_ALIGN: pointer not 16-byte aligned";
    case ZQ_ERR_UNSUPPORTED: return "ZQ_ERR_UNSUPPORTED: request not handled by this build";
    case ZQ_ERR_CUDA: return "ZQ_ERR_CUDA: a CUDA call failed";
    case ZQ_ERR_TIMEOUT: return "ZQ_ERR_TIMEOUT: a kernel gave up a bounded wait";
    default: return "unknown zq status";
  }
}

int zq_abi_version(void) { return 105; }

zq_status zq_set_option(int key, int value) {
  if (key < ZQ_OPT_GEMM_PATH || key > ZQ_OPT_CTA_PAIR) return ZQ_ERR_UNSUPPORTED;
  if (value < 0) return ZQ_ERR_SHAPE;
  if (key == ZQ_OPT_GEMM_PATH && value > 4) return ZQ_ERR_SHAPE;
  if (key == ZQ_OPT_CTA_PAIR && value > 2) return ZQ_ERR_SHAPE;
  if (key == ZQ_OPT_GEMM_BN && value != 0 && (value % 16 != 0 || value > 256)) return ZQ_ERR_SHAPE;
  g_opts[key].store(value, std::memory_order_relaxed);
  return ZQ_OK;
}

int zq_get_option(int key) { return option(key); }

unsigned long long zq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

zq_status zq_device_status(zq_stream_t stream, int* detail) {
  if (detail) *detail = 0;
  ZQ_CUDA_OK(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int v = 0;
  ZQ_CUDA_OK(cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(int)));
  if (v != 0) {
    int zero = 0;
    ZQ_CUDA_OK(cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(int)));
    if (detail) *detail = v;
    return ZQ_ERR_TIMEOUT;
  }
  return ZQ_OK;
}

zq_status zq_debug_wait_timeout(zq_stream_t stream) {
  int* st = device_status_ptr();
  if (!st) return ZQ_ERR_CUDA;
  count_launch();
  debug_wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(st);
  ZQ_CUDA_OK(cudaGetLastError());
  return ZQ_OK;
}

}  // extern "C"
