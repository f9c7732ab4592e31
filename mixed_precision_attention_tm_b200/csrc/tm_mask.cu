// tm_mask.cu -- routing bitmask (tm_build_mask, tm_build_mask_host), the
// content-driven scale policy (tm_build_mask_scale_policy(_varlen),
// tm_key_tile_scales) and routing statistics (tm_route_stats).
//
// TileMix (Lattice paper page), abstract: routing decisions are packed into
// compact bitmasks, one bit per query tile x group of g adjacent key tiles,
// and every legal tile group is routed.  The pages give no policy; this
// builder draws a seeded Bernoulli(p) per legal, non-forced group from the
// SplitMix64 output function (Steele, Lea and Flood, OOPSLA 2014), a
// counter-based hash, so the device kernel and the host twin below produce
// identical bits from the same function.
#include <cuda_runtime.h>

#include <vector>

#include "tm_device.cuh"
#include "tm_host.h"

namespace tmk {
namespace {

struct MaskArgs {
  int Hq;
  int tile_m, tile_n, g;
  int causal;
  double p;
  uint64_t seed;
  int force_diag, force_sink;
  int W;
};

__host__ __device__ inline uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Last key index visible to query row i (bottom-right causal), -1 if none.
__host__ __device__ inline int64_t last_key(int64_t i, int64_t lq, int64_t lk, int causal) {
  if (lk <= 0) return -1;
  if (!causal) return lk - 1;
  const int64_t c = i + lk - lq;
  return c < lk - 1 ? c : lk - 1;
}

// Word w of the bitmask row of query tile I (global index ig) of a sequence
// with lengths lq, lk, for head h.
__host__ __device__ inline uint32_t mask_word(const MaskArgs& a, int h, int64_t ig, int64_t I,
                                              int64_t lq, int64_t lk, int w) {
  const int64_t r0 = I * a.tile_m;
  const int64_t rows = (lq - r0) < a.tile_m ? (lq - r0) : a.tile_m;
  const int64_t jmax = last_key(r0 + rows - 1, lq, lk, a.causal);
  if (jmax < 0) return 0u;
  const int64_t nj = jmax / a.tile_n + 1;
  const int64_t ng = (nj - 1) / a.g + 1;
  const int64_t gdiag = (nj - 1) / a.g;
  uint32_t word = 0u;
  for (int bit = 0; bit < 32; ++bit) {
    const int64_t G = static_cast<int64_t>(w) * 32 + bit;
    if (G >= ng) break;
    if (a.force_diag && G == gdiag) continue;
    if (a.force_sink && G == 0) continue;
    const uint64_t key = (static_cast<uint64_t>(h) << 40) + (static_cast<uint64_t>(ig) << 20) +
                         static_cast<uint64_t>(G);
    const uint64_t u = splitmix64(a.seed ^ key) >> 11;
    const double uf = static_cast<double>(u) * 1.1102230246251565e-16;   // 2^-53, exact
    if (uf < a.p) word |= 1u << bit;
  }
  return word;
}

// One warp per (query tile, sequence, head); lanes stride over the W words.
__global__ void build_mask_kernel(uint32_t* __restrict__ bm, int64_t head_stride,
                                  const int32_t* __restrict__ cu, const int32_t* __restrict__ cu_k,
                                  int64_t Lq, int64_t Lk, int64_t max_lk, MaskArgs a, DevErr err) {
  const int I = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  SeqInfo s = seq_info(cu, b, Lq, a.tile_m);
  const int64_t lq = s.len;
  // key length: from cu_k when the key offsets differ from the query offsets
  const int64_t lk = cu_k ? seq_info(cu_k, b, Lk, a.tile_n).len : (cu ? s.len : Lk);
  if (cu_k != nullptr && lk > max_lk) {   // the row of W words was sized for max_lk
    if (I == 0 && threadIdx.x == 0) dev_error(err, TM_DEVERR_SEQLEN);
    return;
  }
  if (cu != nullptr && I == 0 && threadIdx.x == 0 &&
      lq > static_cast<int64_t>(gridDim.x) * a.tile_m)
    dev_error(err, TM_DEVERR_SEQLEN);
  if (static_cast<int64_t>(I) * a.tile_m >= lq) return;
  const int64_t ig = s.tile_base + I;
  uint32_t* row = bm + static_cast<int64_t>(h) * head_stride + ig * a.W;
  for (int w = threadIdx.x; w < a.W; w += blockDim.x) row[w] = mask_word(a, h, ig, I, lq, lk, w);
}

// Content-driven routing from the tile quantisation scales.  With symmetric
// absmax/127 codes the INT8 score of a tile pair is within
// d * s_q * s_k * (127 + 1/4) of the fp16 score (half a step of rounding per
// element), so a group is routed INT8 when s_q[I] times the largest s_k of
// the group's key tiles that query tile I sees is at most tau.  The product
// is one round-to-nearest fp32 multiply (no contraction) so that the decision
// is reproducible bit for bit.  Legality and forcing as in mask_word.
struct PolicyArgs {
  int Hq, Hkv;
  int tile_m, tile_n, g;
  int causal;
  float tau;
  int force_diag, force_sink;
  int W;
};

__device__ inline uint32_t policy_word(const PolicyArgs& a, int h, int64_t ig, int64_t I, int64_t lq,
                                       int64_t lk, int64_t kbase, const float* qs, const float* ks,
                                       int w) {
  const int64_t r0 = I * a.tile_m;
  const int64_t rows = (lq - r0) < a.tile_m ? (lq - r0) : a.tile_m;
  const int64_t jmax = last_key(r0 + rows - 1, lq, lk, a.causal);
  if (jmax < 0) return 0u;
  const int64_t nj = jmax / a.tile_n + 1;
  const int64_t ng = (nj - 1) / a.g + 1;
  const int64_t gdiag = (nj - 1) / a.g;
  const int hk = h / (a.Hq / a.Hkv);
  const float sq = qs[ig * a.Hq + h];
  uint32_t word = 0u;
  for (int bit = 0; bit < 32; ++bit) {
    const int64_t G = static_cast<int64_t>(w) * 32 + bit;
    if (G >= ng) break;
    if (a.force_diag && G == gdiag) continue;
    if (a.force_sink && G == 0) continue;
    const int64_t j1 = (G + 1) * a.g < nj ? (G + 1) * a.g : nj;
    float mk = 0.f;
    for (int64_t j = G * a.g; j < j1; ++j) mk = fmaxf(mk, ks[(kbase + j) * a.Hkv + hk]);
    if (__fmul_rn(sq, mk) <= a.tau) word |= 1u << bit;
  }
  return word;
}

// cu_k: key offsets when they differ from the query offsets (prefix-cached
// prefill); key tiles are then numbered per key sequence.
__global__ void build_mask_policy_kernel(uint32_t* __restrict__ bm, int64_t head_stride,
                                         const int32_t* __restrict__ cu, const int32_t* __restrict__ cu_k,
                                         int64_t Lq, int64_t Lk, int64_t max_lk, PolicyArgs a,
                                         const float* __restrict__ qs, const float* __restrict__ ks,
                                         DevErr err) {
  const int I = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  SeqInfo s = seq_info(cu, b, Lq, a.tile_m);
  const int64_t lq = s.len;
  const SeqInfo sk = seq_info(cu_k ? cu_k : cu, b, Lk, a.tile_n);
  const int64_t lk = cu_k ? sk.len : (cu ? s.len : Lk);
  if (cu_k != nullptr && lk > max_lk) {   // the row of W words was sized for max_lk
    if (I == 0 && threadIdx.x == 0) dev_error(err, TM_DEVERR_SEQLEN);
    return;
  }
  if (cu != nullptr && I == 0 && threadIdx.x == 0 &&
      lq > static_cast<int64_t>(gridDim.x) * a.tile_m)
    dev_error(err, TM_DEVERR_SEQLEN);
  if (static_cast<int64_t>(I) * a.tile_m >= lq) return;
  const int64_t kbase = sk.tile_base;
  const int64_t ig = s.tile_base + I;
  uint32_t* row = bm + static_cast<int64_t>(h) * head_stride + ig * a.W;
  for (int w = threadIdx.x; w < a.W; w += blockDim.x) row[w] = policy_word(a, h, ig, I, lq, lk, kbase, qs, ks, w);
}

// Per-token key scales (the fp16 scales of an INT8 cache, [T, Hkv]) reduced
// to one fp32 value per key tile and kv head: the largest scale over the
// tile's tokens.  The scale policy's group statistic is then the largest of
// these over the group's visible key tiles, which equals the largest token
// scale over those tiles' tokens (max is exact and associative).  One block
// of kKeyScaleWarps warps per (key tile, sequence); each warp takes a head.
constexpr int kKeyScaleWarps = 8;

__global__ void __launch_bounds__(32 * kKeyScaleWarps)
key_tile_scale_kernel(float* __restrict__ out, const __half* __restrict__ tok, int Hkv,
                      const int32_t* __restrict__ cu_k, int64_t Lk, int64_t max_lk, int tile_n, DevErr err) {
  const int J = blockIdx.x, b = blockIdx.y;
  const SeqInfo s = seq_info(cu_k, b, Lk, tile_n);
  if (cu_k != nullptr && J == 0 && threadIdx.x == 0 && s.len > max_lk) dev_error(err, TM_DEVERR_SEQLEN);
  if (cu_k != nullptr && s.len > max_lk) return;
  const int64_t r0 = static_cast<int64_t>(J) * tile_n;
  if (r0 >= s.len) return;
  const int64_t rows = (s.len - r0) < tile_n ? (s.len - r0) : tile_n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int h = warp; h < Hkv; h += kKeyScaleWarps) {
    float m = -INFINITY;
    for (int64_t r = lane; r < rows; r += 32)
      m = fmaxf(m, __half2float(tok[(s.start + r0 + r) * Hkv + h]));
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) out[(s.tile_base + J) * Hkv + h] = m;
  }
}

tm_status check_mask_args(int32_t Hq, int32_t tile_m, int32_t tile_n, int32_t g, double p) {
  if (Hq <= 0 || Hq >= (1 << 24)) return TM_ERR_INVALID_ARG;
  if (tile_m <= 0 || tile_n <= 0 || g <= 0) return TM_ERR_INVALID_ARG;
  if (!(p >= 0.0 && p <= 1.0)) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

}  // namespace
}  // namespace tmk

extern "C" {

static tm_status build_mask_impl(uint32_t* bitmask, int32_t Hq, const int32_t* cu_seqlens,
                                 const int32_t* cu_k, int32_t batch, int32_t max_seqlen, int32_t max_k,
                                 int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n,
                        int32_t g, int32_t causal, double p, uint64_t seed, int32_t force_diag,
                        int32_t force_sink, int64_t mask_head_stride, void* stream) {
  using namespace tmk;
  tm_status st = check_mask_args(Hq, tile_m, tile_n, g, p);
  if (st != TM_OK) return st;
  if (bitmask == nullptr || reinterpret_cast<uintptr_t>(bitmask) % 4) return TM_ERR_INVALID_ARG;
  const int64_t maxq = cu_seqlens ? max_seqlen : Lq;
  const int64_t maxk = cu_seqlens ? (cu_k ? max_k : max_seqlen) : Lk;
  if (cu_k != nullptr && (cu_seqlens == nullptr || max_k <= 0)) return TM_ERR_INVALID_ARG;
  if (cu_seqlens != nullptr && (batch <= 0 || max_seqlen <= 0)) return TM_ERR_INVALID_ARG;
  if (maxq < 0 || maxk < 0) return TM_ERR_INVALID_ARG;
  MaskArgs a{Hq, tile_m, tile_n, g, causal ? 1 : 0, p, seed, force_diag ? 1 : 0,
             force_sink ? 1 : 0, tm_mask_words(maxk, tile_n, g)};
  const int64_t nqt_max = (maxq + tile_m - 1) / tile_m;
  if (nqt_max == 0) return TM_OK;
  if (mask_head_stride < 0) return TM_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr && Hq > 1 && mask_head_stride < nqt_max * a.W) return TM_ERR_INVALID_ARG;
  const int nb = cu_seqlens ? batch : 1;
  if (nqt_max > 0x7fffffff || nb > 65535 || Hq > 65535) return TM_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(nqt_max), static_cast<unsigned>(nb), static_cast<unsigned>(Hq));
  DevErr err{device_error_word()};
  build_mask_kernel<<<grid, 32, 0, as_stream(stream)>>>(bitmask, mask_head_stride, cu_seqlens, cu_k, Lq,
                                                        Lk, maxk, a, err);
  return check_cuda(cudaGetLastError());
}

tm_status tm_build_mask(uint32_t* bitmask, int32_t Hq, const int32_t* cu_seqlens, int32_t batch,
                        int32_t max_seqlen, int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n,
                        int32_t g, int32_t causal, double p, uint64_t seed, int32_t force_diag,
                        int32_t force_sink, int64_t mask_head_stride, void* stream) {
  return build_mask_impl(bitmask, Hq, cu_seqlens, nullptr, batch, max_seqlen, 0, Lq, Lk, tile_m, tile_n, g,
                         causal, p, seed, force_diag, force_sink, mask_head_stride, stream);
}

tm_status tm_build_mask_varlen(uint32_t* bitmask, int32_t Hq, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, int32_t batch, int32_t max_seqlen_q,
                               int32_t max_seqlen_k, int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                               double p, uint64_t seed, int32_t force_diag, int32_t force_sink,
                               int64_t mask_head_stride, void* stream) {
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return TM_ERR_INVALID_ARG;
  return build_mask_impl(bitmask, Hq, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q, max_seqlen_k, 0, 0, tile_m,
                         tile_n, g, causal, p, seed, force_diag, force_sink, mask_head_stride, stream);
}

static tm_status scale_policy_impl(uint32_t* bitmask, int32_t Hq, int32_t Hkv, const int32_t* cu_seqlens,
                                   const int32_t* cu_k, int32_t batch, int32_t max_seqlen, int32_t max_k,
                                   int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n, int32_t g,
                                   int32_t causal, const float* q_scales, const float* k_scales, float tau,
                                   int32_t force_diag, int32_t force_sink, int64_t mask_head_stride,
                                   void* stream) {
  using namespace tmk;
  tm_status st = check_mask_args(Hq, tile_m, tile_n, g, 0.5);
  if (st != TM_OK) return st;
  if (Hkv <= 0 || Hq % Hkv != 0) return TM_ERR_INVALID_ARG;
  if (tau != tau) return TM_ERR_INVALID_ARG;   // NaN
  if (bitmask == nullptr || reinterpret_cast<uintptr_t>(bitmask) % 4) return TM_ERR_INVALID_ARG;
  if (q_scales == nullptr || k_scales == nullptr) return TM_ERR_INVALID_ARG;
  const int64_t maxq = cu_seqlens ? max_seqlen : Lq;
  const int64_t maxk = cu_seqlens ? (cu_k ? max_k : max_seqlen) : Lk;
  if (cu_k != nullptr && (cu_seqlens == nullptr || max_k <= 0)) return TM_ERR_INVALID_ARG;
  if (cu_seqlens != nullptr && (batch <= 0 || max_seqlen <= 0)) return TM_ERR_INVALID_ARG;
  if (maxq < 0 || maxk < 0) return TM_ERR_INVALID_ARG;
  PolicyArgs a{Hq, Hkv, tile_m, tile_n, g, causal ? 1 : 0, tau, force_diag ? 1 : 0, force_sink ? 1 : 0,
               tm_mask_words(maxk, tile_n, g)};
  const int64_t nqt_max = (maxq + tile_m - 1) / tile_m;
  if (nqt_max == 0) return TM_OK;
  if (mask_head_stride < 0) return TM_ERR_INVALID_ARG;
  if (cu_seqlens == nullptr && Hq > 1 && mask_head_stride < nqt_max * a.W) return TM_ERR_INVALID_ARG;
  const int nb = cu_seqlens ? batch : 1;
  if (nqt_max > 0x7fffffff || nb > 65535 || Hq > 65535) return TM_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(nqt_max), static_cast<unsigned>(nb), static_cast<unsigned>(Hq));
  DevErr err{device_error_word()};
  build_mask_policy_kernel<<<grid, 32, 0, as_stream(stream)>>>(bitmask, mask_head_stride, cu_seqlens, cu_k, Lq,
                                                               Lk, maxk, a, q_scales, k_scales, err);
  return check_cuda(cudaGetLastError());
}

tm_status tm_build_mask_scale_policy(uint32_t* bitmask, int32_t Hq, int32_t Hkv, const int32_t* cu_seqlens,
                                     int32_t batch, int32_t max_seqlen, int64_t Lq, int64_t Lk, int32_t tile_m,
                                     int32_t tile_n, int32_t g, int32_t causal, const float* q_scales,
                                     const float* k_scales, float tau, int32_t force_diag, int32_t force_sink,
                                     int64_t mask_head_stride, void* stream) {
  return scale_policy_impl(bitmask, Hq, Hkv, cu_seqlens, nullptr, batch, max_seqlen, 0, Lq, Lk, tile_m, tile_n, g,
                           causal, q_scales, k_scales, tau, force_diag, force_sink, mask_head_stride, stream);
}

tm_status tm_build_mask_scale_policy_varlen(uint32_t* bitmask, int32_t Hq, int32_t Hkv,
                                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                            int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                            int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                                            const float* q_scales, const float* k_scales, float tau,
                                            int32_t force_diag, int32_t force_sink, int64_t mask_head_stride,
                                            void* stream) {
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return TM_ERR_INVALID_ARG;
  return scale_policy_impl(bitmask, Hq, Hkv, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q, max_seqlen_k, 0, 0,
                           tile_m, tile_n, g, causal, q_scales, k_scales, tau, force_diag, force_sink,
                           mask_head_stride, stream);
}

tm_status tm_key_tile_scales(float* k_tile_scales, const void* k_token_scales, int32_t Hkv,
                             const int32_t* cu_seqlens_k, int32_t batch, int32_t max_seqlen_k, int64_t Lk,
                             int32_t tile_n, void* stream) {
  using namespace tmk;
  if (k_tile_scales == nullptr || k_token_scales == nullptr) return TM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(k_tile_scales) % 4 || reinterpret_cast<uintptr_t>(k_token_scales) % 2)
    return TM_ERR_INVALID_ARG;
  if (Hkv <= 0 || tile_n <= 0) return TM_ERR_INVALID_ARG;
  if (cu_seqlens_k != nullptr && (batch <= 0 || max_seqlen_k < 0)) return TM_ERR_INVALID_ARG;
  const int64_t maxk = cu_seqlens_k ? max_seqlen_k : Lk;
  if (maxk < 0) return TM_ERR_INVALID_ARG;
  const int64_t nkt_max = (maxk + tile_n - 1) / tile_n;
  if (nkt_max == 0) return TM_OK;
  const int nb = cu_seqlens_k ? batch : 1;
  if (nkt_max > 0x7fffffff || nb > 65535) return TM_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(nkt_max), static_cast<unsigned>(nb));
  DevErr err{device_error_word()};
  key_tile_scale_kernel<<<grid, 32 * kKeyScaleWarps, 0, as_stream(stream)>>>(
      k_tile_scales, static_cast<const __half*>(k_token_scales), Hkv, cu_seqlens_k, Lk, maxk, tile_n, err);
  return check_cuda(cudaGetLastError());
}

tm_status tm_build_mask_host(uint32_t* bitmask_host, int32_t Hq, const int32_t* cu_seqlens_host,
                             int32_t batch, int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n,
                             int32_t g, int32_t causal, double p, uint64_t seed,
                             int32_t force_diag, int32_t force_sink) {
  using namespace tmk;
  tm_status st = check_mask_args(Hq, tile_m, tile_n, g, p);
  if (st != TM_OK) return st;
  if (bitmask_host == nullptr) return TM_ERR_INVALID_ARG;
  const int nb = cu_seqlens_host ? batch : 1;
  if (cu_seqlens_host && batch <= 0) return TM_ERR_INVALID_ARG;
  int64_t maxk = Lk;
  if (cu_seqlens_host) {
    maxk = 0;
    for (int b = 0; b < nb; ++b) {
      const int64_t len = static_cast<int64_t>(cu_seqlens_host[b + 1]) - cu_seqlens_host[b];
      if (len < 0) return TM_ERR_INVALID_ARG;
      if (len > maxk) maxk = len;
    }
  }
  MaskArgs a{Hq, tile_m, tile_n, g, causal ? 1 : 0, p, seed, force_diag ? 1 : 0,
             force_sink ? 1 : 0, tm_mask_words(maxk, tile_n, g)};
  const int64_t nqt = tm_count_tiles(cu_seqlens_host, batch, Lq, tile_m);
  if (nqt < 0) return TM_ERR_INVALID_ARG;
  const int64_t hs = nqt * a.W;
  for (int h = 0; h < Hq; ++h) {
    int64_t ig = 0;
    for (int b = 0; b < nb; ++b) {
      const int64_t lq = cu_seqlens_host ? cu_seqlens_host[b + 1] - cu_seqlens_host[b] : Lq;
      const int64_t lk = cu_seqlens_host ? lq : Lk;
      const int64_t n = (lq + tile_m - 1) / tile_m;
      for (int64_t I = 0; I < n; ++I, ++ig)
        for (int w = 0; w < a.W; ++w)
          bitmask_host[h * hs + ig * a.W + w] = mask_word(a, h, ig, I, lq, lk, w);
    }
  }
  return TM_OK;
}

static tm_status route_stats_impl(const uint32_t* bitmask_host, int64_t mask_head_stride, int32_t Hq,
                                  const int32_t* cu_seqlens_host, const int32_t* cu_k_host, int32_t batch,
                                  int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n, int32_t g,
                                  int32_t causal, double* n_vis, double* e8) {
  using namespace tmk;
  if (cu_k_host != nullptr && cu_seqlens_host == nullptr) return TM_ERR_INVALID_ARG;
  const int32_t* ck = cu_k_host ? cu_k_host : cu_seqlens_host;   // key offsets
  if (n_vis == nullptr || e8 == nullptr || Hq <= 0 || tile_m <= 0 || tile_n <= 0 || g <= 0)
    return TM_ERR_INVALID_ARG;
  const int nb = cu_seqlens_host ? batch : 1;
  if (cu_seqlens_host && batch <= 0) return TM_ERR_INVALID_ARG;
  int64_t maxk = Lk;
  if (cu_seqlens_host) {
    maxk = 0;
    for (int b = 0; b < nb; ++b) maxk = std::max<int64_t>(maxk, ck[b + 1] - ck[b]);
  }
  const int W = tm_mask_words(maxk, tile_n, g);
  long double nv = 0, ne8 = 0;
  int64_t ig = 0;
  std::vector<int64_t> per_tile;
  for (int b = 0; b < nb; ++b) {
    const int64_t lq = cu_seqlens_host ? cu_seqlens_host[b + 1] - cu_seqlens_host[b] : Lq;
    const int64_t lk = cu_seqlens_host ? ck[b + 1] - ck[b] : Lk;
    const int64_t n = (lq + tile_m - 1) / tile_m;
    for (int64_t I = 0; I < n; ++I, ++ig) {
      const int64_t r0 = I * tile_m;
      const int64_t rows = std::min<int64_t>(tile_m, lq - r0);
      const int64_t jmax = last_key(r0 + rows - 1, lq, lk, causal);
      if (jmax < 0) continue;
      const int64_t nj = jmax / tile_n + 1;
      per_tile.assign(static_cast<size_t>(nj), 0);
      int64_t tile_vis = 0;
      for (int64_t r = 0; r < rows; ++r) {
        const int64_t lim = last_key(r0 + r, lq, lk, causal);
        if (lim < 0) continue;
        tile_vis += lim + 1;
        for (int64_t J = 0; J * tile_n <= lim; ++J)
          per_tile[J] += std::min<int64_t>(tile_n, lim - J * tile_n + 1);
      }
      nv += static_cast<long double>(tile_vis) * Hq;
      if (bitmask_host == nullptr) continue;
      for (int h = 0; h < Hq; ++h) {
        const uint32_t* row = bitmask_host + h * mask_head_stride + ig * W;
        for (int64_t J = 0; J < nj; ++J) {
          const int64_t G = J / g;
          if ((row[G >> 5] >> (G & 31)) & 1u) ne8 += per_tile[J];
        }
      }
    }
  }
  *n_vis = static_cast<double>(nv);
  *e8 = static_cast<double>(ne8);
  return TM_OK;
}

tm_status tm_route_stats(const uint32_t* bitmask_host, int64_t mask_head_stride, int32_t Hq,
                         const int32_t* cu_seqlens_host, int32_t batch, int64_t Lq, int64_t Lk,
                         int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal, double* n_vis,
                         double* e8) {
  return route_stats_impl(bitmask_host, mask_head_stride, Hq, cu_seqlens_host, nullptr, batch, Lq, Lk, tile_m,
                          tile_n, g, causal, n_vis, e8);
}

tm_status tm_route_stats_varlen(const uint32_t* bitmask_host, int64_t mask_head_stride, int32_t Hq,
                                const int32_t* cu_seqlens_q_host, const int32_t* cu_seqlens_k_host,
                                int32_t batch, int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                                double* n_vis, double* e8) {
  if (cu_seqlens_q_host == nullptr || cu_seqlens_k_host == nullptr) return TM_ERR_INVALID_ARG;
  return route_stats_impl(bitmask_host, mask_head_stride, Hq, cu_seqlens_q_host, cu_seqlens_k_host, batch, 0, 0,
                          tile_m, tile_n, g, causal, n_vis, e8);
}

}  // extern "C"
