// tm_cache_expand.cu -- the INT8 K/V cache expanded once per step into a
// caller-owned workspace (tm_cache_workspace_bytes, and the expansion that
// tm_attn_fwd_cache_ws runs before its attention launch).
//
// TileMix (Lattice paper page), abstract: the method supports INT8 K/V
// caches; FP16-routed groups and P.V read the cache's fp16 view
// fp16(code * scale), INT8-routed groups its K codes with the scale of each
// key.  In prefill every K / V tile of a KV head is read by every query tile
// of every query head in its group, so the fp16 view is written once here,
// HBM-bound, instead of being recomputed in shared memory by each CTA that
// reads it.  The per-token K scales are rewritten alongside as fp32 (exact),
// one row of 128 values per key tile and KV head, so that the attention
// kernel can bring a key tile's scales with one aligned bulk copy.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tm_attn_internal.h"
#include "tm_device.cuh"
#include "tm_host.h"

namespace tmk {
namespace {

constexpr int kExpandThreads = 256;

// 16 INT8 codes -> 16 fp16 values fp16_rn(code * scale), exactly: XOR 0x80
// makes code + 128 a byte that, under the fp16 exponent byte 0x64, reads as
// 1024 + code + 128; subtracting 1152 leaves the code exactly, and one fp16
// multiply rounds the exact product once.
__device__ __forceinline__ void expand16(uint4 c, __half2 s2, uint4& lo, uint4& hi) {
  const __half2 bias = __float2half2_rn(1152.0f);
  const uint32_t w[4] = {c.x ^ 0x80808080u, c.y ^ 0x80808080u, c.z ^ 0x80808080u, c.w ^ 0x80808080u};
  uint32_t o[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t a = __byte_perm(w[q], 0x64646464u, 0x4140u);   // bytes b0, 0x64, b1, 0x64
    uint32_t b = __byte_perm(w[q], 0x64646464u, 0x4342u);   // bytes b2, 0x64, b3, 0x64
    __half2 va = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&a), bias), s2);
    __half2 vb = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&b), bias), s2);
    o[2 * q] = *reinterpret_cast<uint32_t*>(&va);
    o[2 * q + 1] = *reinterpret_cast<uint32_t*>(&vb);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// One block per (key tile J, sequence b): the tile's tokens for every KV head
// of K and V, and the tile's row of per-token K scales for every KV head
// (rows past the sequence's end get 0).  d = 128: 8 chunks of 16 codes per
// (token, head).
__global__ void __launch_bounds__(kExpandThreads)
cache_expand_kernel(const uint8_t* __restrict__ kc, const __half* __restrict__ ks, const uint8_t* __restrict__ vc,
                    const __half* __restrict__ vs, __half* __restrict__ k16, __half* __restrict__ v16,
                    float* __restrict__ kst, int Hkv, const int32_t* __restrict__ cu_k, int64_t Lk, int64_t max_lk,
                    int64_t kst_tiles, DevErr err) {
  const int J = blockIdx.x, b = blockIdx.y;
  const SeqInfo s = seq_info(cu_k, b, Lk, 128);
  if (cu_k != nullptr && s.len > max_lk) {   // the grid was sized for max_lk
    if (J == 0 && threadIdx.x == 0) dev_error(err, TM_DEVERR_SEQLEN);
    return;
  }
  const int64_t r0 = static_cast<int64_t>(J) * 128;
  if (r0 >= s.len) return;
  if (s.tile_base + J >= kst_tiles) {   // more key tiles than the workspace was laid out for
    if (threadIdx.x == 0) dev_error(err, TM_DEVERR_SEQLEN);
    return;
  }
  const int rows = static_cast<int>(s.len - r0 < 128 ? s.len - r0 : 128);
  const int64_t tok0 = s.start + r0;
  const int chunks = rows * Hkv * 8;
  for (int c = threadIdx.x; c < chunks; c += kExpandThreads) {
    const int64_t th = tok0 * Hkv + (c >> 3);   // (token, head) index
    const int64_t e = th * 128 + (c & 7) * 16;  // first element of the chunk
    uint4 lo, hi;
    expand16(__ldcs(reinterpret_cast<const uint4*>(kc + e)), __half2half2(ks[th]), lo, hi);
    *reinterpret_cast<uint4*>(k16 + e) = lo;
    *reinterpret_cast<uint4*>(k16 + e + 8) = hi;
    expand16(__ldcs(reinterpret_cast<const uint4*>(vc + e)), __half2half2(vs[th]), lo, hi);
    *reinterpret_cast<uint4*>(v16 + e) = lo;
    *reinterpret_cast<uint4*>(v16 + e + 8) = hi;
  }
  for (int i = threadIdx.x; i < Hkv * 128; i += kExpandThreads) {
    const int h = i >> 7, r = i & 127;
    kst[(static_cast<int64_t>(h) * kst_tiles + s.tile_base + J) * 128 + r] =
        r < rows ? __half2float(ks[(tok0 + r) * Hkv + h]) : 0.f;
  }
}

int64_t round256(int64_t x) { return (x + 255) / 256 * 256; }

}  // namespace

CacheWsLayout cache_ws_layout(int64_t Tk, int32_t Hkv, int32_t batch) {
  CacheWsLayout L;
  L.kst_tiles = (Tk + 127) / 128 + (batch > 0 ? batch : 0);
  const int64_t kv = round256(Tk * Hkv * 128 * 2);
  L.off_k16 = 0;
  L.off_v16 = kv;
  L.off_kst = 2 * kv;
  L.bytes = 2 * kv + round256(static_cast<int64_t>(Hkv) * L.kst_tiles * 128 * 4);
  return L;
}

tm_status launch_cache_expand(const tm_tensor* k, const tm_tensor* v, const int32_t* cu_k, int32_t batch,
                              int32_t max_k, void* workspace, const CacheWsLayout& L, cudaStream_t stream) {
  const int64_t maxk = cu_k ? max_k : k->T;
  const int64_t nkt = (maxk + 127) / 128;
  const int nb = cu_k ? batch : 1;
  if (nkt == 0) return TM_OK;
  if (nkt > 0x7fffffff || nb > 65535) return TM_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  dim3 grid(static_cast<unsigned>(nkt), static_cast<unsigned>(nb));
  cache_expand_kernel<<<grid, kExpandThreads, 0, stream>>>(
      reinterpret_cast<const uint8_t*>(k->codes), static_cast<const __half*>(k->scales),
      reinterpret_cast<const uint8_t*>(v->codes), static_cast<const __half*>(v->scales),
      reinterpret_cast<__half*>(ws + L.off_k16), reinterpret_cast<__half*>(ws + L.off_v16),
      reinterpret_cast<float*>(ws + L.off_kst), static_cast<int>(k->H), cu_k, k->T, maxk, L.kst_tiles,
      DevErr{device_error_word()});
  return check_cuda(cudaGetLastError());
}

}  // namespace tmk

extern "C" int64_t tm_cache_workspace_bytes(int64_t Tk, int32_t Hkv, int32_t batch) {
  if (Tk < 0 || Hkv <= 0 || batch < 0) return -1;
  return tmk::cache_ws_layout(Tk, Hkv, batch).bytes;
}
