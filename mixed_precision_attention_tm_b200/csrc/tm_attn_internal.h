// tm_attn_internal.h -- launchers shared between the attention translation
// units (not part of the C ABI).
#pragma once

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

// One 128-row query tile per CTA with two score buffers in TMEM and the keys
// of each score tile split between two softmax warpgroups (d = 128).
tm_status launch_attn_split(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                            cudaStream_t stream);

// INT8 K/V cache (codes + per-token fp16 scales), d = 128, 128-key tiles.
tm_status launch_attn_cache(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t tile_m, int32_t g,
                            int32_t causal, cudaStream_t stream);

}  // namespace tmk
