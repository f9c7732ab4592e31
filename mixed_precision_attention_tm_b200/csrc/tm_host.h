// tm_host.h -- host-side helpers shared by the libtm translation units:
// status bookkeeping, the per-device error word, and TMA descriptor encoding
// through the driver entry point (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tm.h"

namespace tmk {

// Records a failed CUDA call for tm_last_cuda_error() and maps it to a status.
tm_status cuda_fail(int code);

inline tm_status check_cuda(cudaError_t e) {
  return e == cudaSuccess ? TM_OK : cuda_fail(static_cast<int>(e));
}

// Device address of this device's error word (set up on first use).
unsigned int* device_error_word();

// cuTensorMapEncodeTiled for a rank-3 [T, H, d] tensor (d innermost), box
// {box_d, 1, box_rows}, with the given swizzle.  Out-of-range rows read 0.
tm_status encode_thd_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                         int elem_bytes, int64_t T, int64_t H, int64_t d, int64_t stride_t,
                         int64_t stride_h, int box_d, int box_rows, CUtensorMapSwizzle swz);

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace tmk
