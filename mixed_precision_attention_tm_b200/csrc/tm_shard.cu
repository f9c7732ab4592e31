// tm_shard.cu -- reassembly of a prefill output that was split by query
// heads over the ranks of a process group.
//
// Query heads are independent in attention (grouped-query heads share only
// their K / V), so one prefill problem shards over GPUs by blocks of
// consecutive query heads with no exchange on the data path.  A caller that
// wants the whole [T, Hq, d] output on every rank gathers the ranks' slices
// with one all-gather of equal-size buffers [T, h_cap, d] (h_cap = the largest
// shard) and then interleaves them back into token-major order here: row t of
// the output is rank 0's heads of row t, then rank 1's, and so on.  Each
// rank's piece of a row is contiguous on both sides, so the copy is a set of
// 2-D strided copies, one per rank, moved in 16-byte vectors.
#include <cuda_runtime.h>

#include "tm_host.h"

namespace tmk {
namespace {

constexpr int kMaxWorld = 64;

struct MergeArgs {
  int64_t T;
  int64_t out_stride_t;   // elements between output rows
  int64_t src_stride_t;   // h_cap * d elements between rows of one rank's slice
  int64_t src_rank;       // T * h_cap * d elements between ranks' slices
  int32_t d;
  int32_t head_start[kMaxWorld + 1];
};

// blockIdx.y = rank; the x dimension strides over (row, 16-byte chunk) pairs
// of that rank's piece, chunk fastest so consecutive threads touch
// consecutive addresses on both sides.
__global__ void __launch_bounds__(256) merge_head_shards_kernel(uint4* __restrict__ out,
                                                                const uint4* __restrict__ src,
                                                                MergeArgs a) {
  const int r = blockIdx.y;
  const int64_t h0 = a.head_start[r];
  const int64_t chunks = (a.head_start[r + 1] - h0) * a.d / 8;  // 16-byte chunks per row
  if (chunks == 0) return;
  const int64_t total = a.T * chunks;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += step) {
    const int64_t t = i / chunks;
    const int64_t c = i - t * chunks;
    // element offsets / 8 = uint4 offsets (all strides are multiples of 8)
    const int64_t s = (r * a.src_rank + t * a.src_stride_t) / 8 + c;
    const int64_t o = (t * a.out_stride_t + h0 * a.d) / 8 + c;
    out[o] = __ldg(src + s);
  }
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  return sms;
}

}  // namespace
}  // namespace tmk

extern "C" tm_status tm_merge_head_shards(void* out, int64_t out_stride_t, const void* gathered, int64_t T,
                                          int32_t Hq, int32_t d, int32_t world, int32_t h_cap,
                                          const int32_t* head_start, void* stream) {
  using namespace tmk;
  if (head_start == nullptr || T < 0 || Hq <= 0 || d <= 0 || (d % 8) != 0) return TM_ERR_INVALID_ARG;
  if (world < 1 || world > kMaxWorld || h_cap < 1) return TM_ERR_INVALID_ARG;
  if (head_start[0] != 0 || head_start[world] != Hq) return TM_ERR_INVALID_ARG;
  for (int r = 0; r < world; ++r) {
    const int32_t n = head_start[r + 1] - head_start[r];
    if (n < 0 || n > h_cap) return TM_ERR_INVALID_ARG;
  }
  if (out_stride_t < static_cast<int64_t>(Hq) * d || (out_stride_t % 8) != 0) return TM_ERR_INVALID_ARG;
  if (T == 0) return TM_OK;
  if (out == nullptr || gathered == nullptr) return TM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(out) & 15u) || (reinterpret_cast<uintptr_t>(gathered) & 15u))
    return TM_ERR_INVALID_ARG;
  MergeArgs a;
  a.T = T;
  a.out_stride_t = out_stride_t;
  a.src_stride_t = static_cast<int64_t>(h_cap) * d;
  a.src_rank = T * a.src_stride_t;
  a.d = d;
  for (int r = 0; r <= kMaxWorld; ++r) a.head_start[r] = r <= world ? head_start[r] : Hq;
  // enough blocks for every SM to hold several, spread over the ranks
  const int64_t per_rank = (T * h_cap * (d / 8) + 255) / 256;
  const int64_t want = (static_cast<int64_t>(sm_count()) * 8 + world - 1) / world;
  const unsigned bx = static_cast<unsigned>(per_rank < want ? (per_rank > 0 ? per_rank : 1) : want);
  merge_head_shards_kernel<<<dim3(bx, static_cast<unsigned>(world)), 256, 0, as_stream(stream)>>>(
      static_cast<uint4*>(out), static_cast<const uint4*>(gathered), a);
  return check_cuda(cudaGetLastError());
}
