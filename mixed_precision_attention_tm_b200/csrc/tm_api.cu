// tm_api.cu -- shared C-ABI entry points of libtm (status strings, version,
// device error word) and the host helpers declared in tm_host.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tm_device.cuh"
#include "tm_host.h"

namespace {

thread_local int g_last_cuda_error = 0;

// One word per device; bit TM_DEVERR_* set by kernels with atomicOr.
__device__ unsigned int g_error_word;

constexpr int kMaxDevices = 64;
unsigned int* g_error_ptr[kMaxDevices] = {};
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// One thread waits, with the library's bounded wait, on an mbarrier that
// nothing arrives on; the wait gives up after limit_ns and records
// TM_DEVERR_TIMEOUT.  No copy or MMA is in flight, so the kernel just returns.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, tmk::DevErr err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  tmk::mbar_init(tmk::smem_u32(&bar), 1);
  abort_flag = 0;
  tmk::fence_barrier_init();
  tmk::mbar_wait_limit(tmk::smem_u32(&bar), 0, err, &abort_flag, limit_ns);
}

}  // namespace

namespace tmk {

tm_status cuda_fail(int code) {
  g_last_cuda_error = code;
  return TM_ERR_CUDA;
}

unsigned int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_error_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_error_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_error_ptr[dev];
}

tm_status encode_thd_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         int elem_bytes, int64_t T, int64_t H, int64_t d, int64_t stride_t,
                         int64_t stride_h, int box_d, int box_rows, CUtensorMapSwizzle swz) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || fn == nullptr || q != cudaDriverEntryPointSuccess)
        return cuda_fail(e != cudaSuccess ? static_cast<int>(e) : -1);
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride_h * elem_bytes),
                           static_cast<cuuint64_t>(stride_t * elem_bytes)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), 1u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = g_encode(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(1000 + static_cast<int>(r));
  return TM_OK;
}

}  // namespace tmk

extern "C" {

const char* tm_status_string(tm_status s) {
  switch (s) {
    case TM_OK: return "ok";
    case TM_ERR_INVALID_ARG: return "invalid argument";
    case TM_ERR_UNSUPPORTED: return "unsupported configuration";
    case TM_ERR_CUDA: return "CUDA error";
    case TM_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int32_t tm_last_cuda_error(void) { return g_last_cuda_error; }

const char* tm_version(void) { return "0.1.0"; }

tm_status tm_get_device_error(void* stream) {
  unsigned int* w = tmk::device_error_word();
  if (w == nullptr) return tmk::cuda_fail(static_cast<int>(cudaErrorInvalidSymbol));
  cudaStream_t s = tmk::as_stream(stream);
  unsigned int host = 0;
  tm_status st = tmk::check_cuda(cudaMemcpyAsync(&host, w, sizeof(host), cudaMemcpyDeviceToHost, s));
  if (st != TM_OK) return st;
  st = tmk::check_cuda(cudaStreamSynchronize(s));
  if (st != TM_OK) return st;
  if (host != 0) {
    st = tmk::check_cuda(cudaMemsetAsync(w, 0, sizeof(unsigned int), s));
    if (st != TM_OK) return st;
    st = tmk::check_cuda(cudaStreamSynchronize(s));
    if (st != TM_OK) return st;
  }
  if (host & 1u) return TM_ERR_TIMEOUT;
  if (host & 2u) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

tm_status tm_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return TM_ERR_INVALID_ARG;
  tmk::DevErr err{tmk::device_error_word()};
  if (err.word == nullptr) return tmk::cuda_fail(static_cast<int>(cudaErrorInvalidSymbol));
  wait_timeout_selftest_kernel<<<1, 32, 0, tmk::as_stream(stream)>>>(limit_ns, err);
  return tmk::check_cuda(cudaGetLastError());
}

int32_t tm_mask_words(int64_t max_lk, int32_t tile_n, int32_t g) {
  if (max_lk < 0 || tile_n <= 0 || g <= 0) return -1;
  const int64_t nkt = (max_lk + tile_n - 1) / tile_n;
  const int64_t ng = (nkt + g - 1) / g;
  const int64_t w = (ng + 31) / 32;
  return static_cast<int32_t>(w < 1 ? 1 : w);
}

int64_t tm_count_tiles(const int32_t* cu_seqlens_host, int32_t batch, int64_t L, int32_t tile) {
  if (tile <= 0) return -1;
  if (cu_seqlens_host == nullptr) return L < 0 ? -1 : (L + tile - 1) / tile;
  if (batch < 0) return -1;
  int64_t n = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t len = static_cast<int64_t>(cu_seqlens_host[b + 1]) - cu_seqlens_host[b];
    if (len < 0) return -1;
    n += (len + tile - 1) / tile;
  }
  return n;
}

}  // extern "C"
