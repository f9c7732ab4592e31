// tm_probe.cu -- instruction-rate probes behind the secondary bounds of the
// attention kernels (measurement only; nothing here is on the prefill path).
//
// The fused attention spends its non-tensor time on one exp2 per visible
// (query, key) pair and, on INT8-routed tiles, one int32 -> fp32 conversion
// per pair.  These probes measure, on the running GPU:
//   [0] MUFU ex2.approx.f32: SM-clock cycles per warp instruction per SM
//       sub-partition (4 warps per sub-partition, 8 independent chains each);
//   [1] cvt.rn.f32.s32 (the plain int32 -> fp32 conversion), same unit;
//   [2] the exact conversion the kernels use instead (integer add of the bits
//       of 1.5 * 2^23, then one fp32 subtract), cycles per converted value
//       per sub-partition;
//   [3] tcgen05.mma kind::f16 M128 N128 K16, cycles per MMA on one SM
//       (back-to-back from one elected thread, accumulating in TMEM);
//   [4] tcgen05.mma kind::i8 M128 N128 K32, same.
// Every wait is bounded (tm_device.cuh); a probe that fails reports -1.
#include <cuda.h>
#include <cuda_runtime.h>

#include <vector>

#include "tm_device.cuh"
#include "tm_host.h"

namespace tmk {
namespace {

constexpr int kAluIters = 64;      // x 16 x 8 instructions per thread
constexpr int kMmaCount = 4096;    // MMAs per SM in the tensor probes

template <int OP>
__global__ void __launch_bounds__(512, 1) alu_rate_kernel(long long* cycles, float* sink) {
  float a[8];
  uint32_t u[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    a[q] = threadIdx.x * 1e-3f + q * 0.01f;
    u[q] = threadIdx.x * 7u + q;
  }
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < kAluIters; ++it) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (OP == 0) {
          a[q] = ex2_approx(a[q]);
        } else if (OP == 1) {
          float f;
          asm volatile("cvt.rn.f32.s32 %0, %1;" : "=f"(f) : "r"(static_cast<int>(u[q])));
          u[q] = __float_as_uint(f) >> 9;
        } else {
          const float f = __int_as_float(static_cast<int>(u[q]) + 0x4B400000) - 12582912.0f;
          u[q] = __float_as_uint(f) >> 9;
        }
      }
    }
  }
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) s += a[q] + __uint_as_float(u[q]);
  if (s == 1234.5f) sink[threadIdx.x] = s;
  if ((threadIdx.x & 31) == 0) cycles[blockIdx.x * 16 + (threadIdx.x >> 5)] = t1 - t0;
}

// tcgen05 rate: A 32 KB and B 32 KB of zeroed shared memory (128-byte
// swizzled K-major tiles), D in TMEM columns [0, 128).
template <bool I8>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(long long* cycles, DevErr err) {
  extern __shared__ uint8_t raw[];
  const uint32_t rs = smem_u32(raw);
  const uint32_t base = (rs + 1023u) & ~1023u;
  uint8_t* sm = raw + (base - rs);
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tslot;
  __shared__ volatile int abort_flag;
  for (int i = threadIdx.x; i < 65536 / 16; i += blockDim.x) reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    abort_flag = 0;
  }
  fence_async_shared();
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(&tslot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  if (threadIdx.x < 32) {
    const uint32_t A = base, B = base + 32768;
    uint64_t ad[8], bd[8];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t off = I8 ? (kk & 3) * 32 : (kk >> 2) * 16384 + (kk & 3) * 32;
      ad[kk] = smem_desc(A + off, 16, 1024, kSwizzle128);
      bd[kk] = smem_desc(B + off, 16, 1024, kSwizzle128);
    }
    const uint32_t idesc = I8 ? idesc_i8(128, 128) : idesc_f16(128, 128, false);
    long long t0 = 0;
    bool ok = true;
    for (int phase = 0; phase < 2; ++phase) {
      const int groups = phase == 0 ? 8 : kMmaCount / 8;
      if (phase == 1) t0 = clock64();
      if (elect_one()) {
        for (int gi = 0; gi < groups; ++gi) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            if (I8) mma_i8_ss(tmem, ad[kk], bd[kk], idesc, 1u);
            else mma_f16_ss(tmem, ad[kk], bd[kk], idesc, 1u);
          }
        }
        tc_commit(smem_u32(&bar));
      }
      __syncwarp();
      ok = mbar_wait_warp(smem_u32(&bar), phase, err, &abort_flag) && ok;
    }
    const long long t1 = clock64();
    if (threadIdx.x == 0) cycles[blockIdx.x] = ok ? (t1 - t0) : -1;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

constexpr int kMmaSmem = 65536 + 1024;

double median_of(long long* v, int n) {
  // insertion sort of a small array
  for (int i = 1; i < n; ++i)
    for (int j = i; j > 0 && v[j - 1] > v[j]; --j) {
      const long long t = v[j];
      v[j] = v[j - 1];
      v[j - 1] = t;
    }
  return static_cast<double>(v[n / 2]);
}

}  // namespace
}  // namespace tmk

extern "C" int64_t tm_probe_scratch_bytes(void) {
  // one cycle count per warp (16 warps) of up to 1024 SMs, plus a 512-float sink
  return static_cast<int64_t>(sizeof(long long)) * 1024 * 16 + static_cast<int64_t>(sizeof(float)) * 512;
}

extern "C" tm_status tm_probe_rates(double* out, int32_t n_out, void* scratch, int64_t scratch_bytes,
                                    void* stream_ptr) {
  using namespace tmk;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (out == nullptr || n_out < 5 || scratch == nullptr) return TM_ERR_INVALID_ARG;
  if (scratch_bytes < tm_probe_scratch_bytes() || (reinterpret_cast<uintptr_t>(scratch) & 15u) != 0)
    return TM_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  tm_status st = check_cuda(cudaGetDevice(&dev));
  if (st != TM_OK) return st;
  st = check_cuda(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  if (st != TM_OK) return st;
  if (sms <= 0 || sms > 1024) return TM_ERR_UNSUPPORTED;
  long long* d_cyc = static_cast<long long*>(scratch);
  float* d_sink = reinterpret_cast<float*>(d_cyc + 1024 * 16);
  std::vector<long long> hostv(1024 * 16);
  long long* host = hostv.data();
  const int n_alu = sms * 16;
  auto alu = [&](auto kern, int slot, double per_instr_div) -> tm_status {
    for (int rep = 0; rep < 2; ++rep) kern<<<sms, 512, 0, stream>>>(d_cyc, d_sink);
    tm_status s2 = check_cuda(cudaGetLastError());
    if (s2 != TM_OK) return s2;
    s2 = check_cuda(cudaMemcpyAsync(host, d_cyc, sizeof(long long) * n_alu, cudaMemcpyDeviceToHost, stream));
    if (s2 != TM_OK) return s2;
    s2 = check_cuda(cudaStreamSynchronize(stream));
    if (s2 != TM_OK) return s2;
    // 4 warps per sub-partition, 8 x 16 x kAluIters instructions per warp
    out[slot] = median_of(host, n_alu) / (static_cast<double>(kAluIters) * 16 * 8 * 4) / per_instr_div;
    return TM_OK;
  };
  st = alu(alu_rate_kernel<0>, 0, 1.0);
  if (st == TM_OK) st = alu(alu_rate_kernel<1>, 1, 1.0);
  if (st == TM_OK) st = alu(alu_rate_kernel<2>, 2, 1.0);
  auto mma = [&](auto kern, int slot) -> tm_status {
    tm_status s2 = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMmaSmem));
    if (s2 != TM_OK) return s2;
    kern<<<sms, 128, kMmaSmem, stream>>>(d_cyc, DevErr{device_error_word()});
    s2 = check_cuda(cudaGetLastError());
    if (s2 != TM_OK) return s2;
    s2 = check_cuda(cudaMemcpyAsync(host, d_cyc, sizeof(long long) * sms, cudaMemcpyDeviceToHost, stream));
    if (s2 != TM_OK) return s2;
    s2 = check_cuda(cudaStreamSynchronize(stream));
    if (s2 != TM_OK) return s2;
    const double med = median_of(host, sms);
    out[slot] = med < 0 ? -1.0 : med / kMmaCount;
    return TM_OK;
  };
  if (st == TM_OK) st = mma(mma_rate_kernel<false>, 3);
  if (st == TM_OK) st = mma(mma_rate_kernel<true>, 4);
  return st;
}
