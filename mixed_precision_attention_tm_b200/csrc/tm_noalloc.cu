// tm_noalloc.cu -- tm_attn_fwd_routed_noalloc: the routed prefill step
// (quantise Q and K, build the routing mask, fused attention) with its
// intermediate buffers in a fixed, library-owned device array instead of
// caller-allocated memory.
//
// Who needs it: callers that cannot hand the library scratch memory -- for
// example a serving engine that reserves nearly all device memory for its own
// pools at start-up and has no allocator it can lend to a C library, or a
// latency-bound deployment that forbids cudaMalloc after initialisation
// because it can synchronise the device and take unbounded time.  They still
// pass Q, K, V and the output; everything else lives in g_tm_scratch.
//
// The array is TM_NOALLOC_SCRATCH_BYTES of device memory on every GPU that
// loads this library, held until the process exits.  All calls share it:
// calls that overlap on the GPU (different streams, or different host
// threads on one device) race on it, so callers serialise them.
#include <cuda_runtime.h>

#include <mutex>

#include "tm_host.h"

namespace {

static __device__ __align__(256) unsigned char g_tm_scratch[TM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
unsigned char* g_scratch_dev[kMaxDev] = {};
std::mutex g_scratch_mu;

// Device address of g_tm_scratch on the current device (looked up once per
// device; in host code the symbol itself is only a host-side handle).
tm_status scratch_address(unsigned char** out) {
  int dev = 0;
  tm_status st = tmk::check_cuda(cudaGetDevice(&dev));
  if (st != TM_OK) return st;
  if (dev < 0 || dev >= kMaxDev) return TM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    st = tmk::check_cuda(cudaGetSymbolAddress(&p, g_tm_scratch));
    if (st != TM_OK) return st;
    g_scratch_dev[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch_dev[dev];
  return TM_OK;
}

int64_t align256(int64_t x) { return (x + 255) & ~static_cast<int64_t>(255); }

}  // namespace

extern "C" tm_status tm_attn_fwd_routed_noalloc(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v,
                                                tm_tensor* out, int32_t tile_m, int32_t tile_n, int32_t g,
                                                int32_t causal, double p, uint64_t seed, int32_t force_diag,
                                                int32_t force_sink, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return TM_ERR_INVALID_ARG;
  if (q->data == nullptr || k->data == nullptr || v->data == nullptr || out->data == nullptr)
    return TM_ERR_INVALID_ARG;
  if (q->T < 0 || k->T < 0 || q->H <= 0 || k->H <= 0 || g < 1) return TM_ERR_INVALID_ARG;
  if ((tile_m != 64 && tile_m != 128) || (tile_n != 64 && tile_n != 128)) return TM_ERR_UNSUPPORTED;
  if (q->d != 64 && q->d != 128) return TM_ERR_UNSUPPORTED;
  // Scratch layout (256-byte aligned parts): Q codes, K codes, Q scales,
  // K scales, routing mask.
  const int64_t nqt = (q->T + tile_m - 1) / tile_m;
  const int64_t nkt = (k->T + tile_n - 1) / tile_n;
  const int64_t W = tm_mask_words(k->T, tile_n, g);
  const int64_t off_qc = 0;
  const int64_t off_kc = off_qc + align256(q->T * q->H * q->d);
  const int64_t off_qs = off_kc + align256(k->T * k->H * k->d);
  const int64_t off_ks = off_qs + align256(nqt * q->H * 4);
  const int64_t off_m = off_ks + align256(nkt * k->H * 4);
  const int64_t total = off_m + align256(q->H * nqt * W * 4);
  if (total > static_cast<int64_t>(TM_NOALLOC_SCRATCH_BYTES)) return TM_ERR_UNSUPPORTED;

  unsigned char* base = nullptr;
  tm_status st = scratch_address(&base);
  if (st != TM_OK) return st;
  int8_t* qc = reinterpret_cast<int8_t*>(base + off_qc);
  int8_t* kc = reinterpret_cast<int8_t*>(base + off_kc);
  float* qs = reinterpret_cast<float*>(base + off_qs);
  float* ks = reinterpret_cast<float*>(base + off_ks);
  uint32_t* mask = reinterpret_cast<uint32_t*>(base + off_m);

  // Every byte read later is written first (all tiles of Q and K, every mask
  // word of every query-tile row), so nothing needs clearing between calls.
  st = tm_quantize_qk(q, k, qc, qs, kc, ks, nullptr, 0, 0, tile_m, tile_n, stream);
  if (st != TM_OK) return st;
  st = tm_build_mask(mask, static_cast<int32_t>(q->H), nullptr, 0, 0, q->T, k->T, tile_m, tile_n, g, causal, p,
                     seed, force_diag, force_sink, nqt * W, stream);
  if (st != TM_OK) return st;
  tm_tensor qq = *q, kk = *k;
  qq.codes = qc;
  qq.scales = qs;
  qq.scale_kind = TM_SCALE_TILE;
  kk.codes = kc;
  kk.scales = ks;
  kk.scale_kind = TM_SCALE_TILE;
  return tm_attn_fwd(&qq, &kk, v, out, nullptr, 0, 0, mask, nqt * W, tile_m, tile_n, g, causal, stream);
}
