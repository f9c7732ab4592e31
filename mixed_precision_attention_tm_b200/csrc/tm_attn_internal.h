// tm_attn_internal.h -- launchers shared between the attention translation
// units (not part of the C ABI).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/tm.h"

namespace tmk {

// Two 128-row query tiles per CTA, 128-key tiles, fp16 K/V (d = 64 or 128).
// cu / cu_k: query / key offsets per sequence (cu_k null: same as cu);
// max_q / max_k: longest query / key sequence.
tm_status launch_attn_pair(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                           const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                           const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                           cudaStream_t stream);

// The FP8 route on the two-query-tile kernel, for launches without an INT8
// plane: q / k carry the FP8 E4M3 codes and tile scales in their codes /
// scales fields; bitmask_fp8 is the FP8 bit plane (d = 128, 128 x 128 tiles).
tm_status launch_attn_pair_fp8(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                               const int32_t* cu, int32_t batch, int32_t max_q, const uint32_t* bitmask_fp8,
                               int64_t mask_hs, int32_t g, int32_t causal, cudaStream_t stream);

// The FP8 third precision: a second routing bit plane (layout of the INT8
// bitmask) and the E4M3 codes and tile scales of Q and K.
struct Fp8Route {
  const uint32_t* bitmask;
  const uint8_t* q_codes;
  const float* q_scales;
  const uint8_t* k_codes;
  const float* k_scales;
};

// One 128-row query tile per CTA with three score buffers in TMEM: at d = 128
// the keys of each score tile are split between two softmax warpgroups, at
// d = 64 the warpgroups take alternate key tiles (two softmax streams).
// f8: the FP8 route, d = 128 only (null or a null bitmask: FP16 / INT8 only).
tm_status launch_attn_split(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                            cudaStream_t stream, const Fp8Route* f8 = nullptr);

// INT8 K/V cache on the two-query-tile kernel: d = 128, 128-row query tiles
// and 128-key tiles; a dequantisation warpgroup writes the fp16 tiles.
tm_status launch_attn_pair_cache(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                                 const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q,
                                 int32_t max_k, const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                                 cudaStream_t stream);

// Workspace of the expanded INT8 cache (tm_cache_expand.cu): the fp16 view of
// K and of V [Tk, Hkv, 128] and the per-token K scales [Hkv][kst_tiles][128]
// fp32, each part 256-byte aligned.  kst_tiles bounds the key tiles of all
// sequences: ceil(Tk / 128) plus one per sequence (batch = 0: one sequence).
struct CacheWsLayout {
  int64_t kst_tiles;
  int64_t off_k16, off_v16, off_kst;
  int64_t bytes;
};
CacheWsLayout cache_ws_layout(int64_t Tk, int32_t Hkv, int32_t batch);

// Writes the workspace from the cache k / v (codes + per-token fp16 scales,
// d = 128).  cu_k: key offsets (null: one sequence of k->T keys).
tm_status launch_cache_expand(const tm_tensor* k, const tm_tensor* v, const int32_t* cu_k, int32_t batch,
                              int32_t max_k, void* workspace, const CacheWsLayout& L, cudaStream_t stream);

// INT8 K/V cache expanded into a workspace: k / v are the cache's fp16 view
// (k's codes field the cache's K codes), the INT8 route's key scales per
// token from kst_ws [Hkv][kst_tiles][128] fp32; routed launches, d = 128,
// 128 x 128 tiles, two query tiles per CTA.
tm_status launch_attn_pair_toks(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                                const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                                const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                                const float* kst_ws, int64_t kst_tiles, cudaStream_t stream);

// INT8 K/V cache (codes + per-token fp16 scales), d = 128, 128-key tiles, one
// query tile per CTA.
tm_status launch_attn_cache(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t tile_m, int32_t g,
                            int32_t causal, cudaStream_t stream);

}  // namespace tmk
