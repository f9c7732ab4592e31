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

#include "tm_host.h"

namespace {

static __device__ __align__(256) unsigned char g_tm_scratch[TM_NOALLOC_SCRATCH_BYTES];

// Device address of g_tm_scratch in the current device's context.  In host
// code the symbol itself is only a host-side handle, so it is resolved here,
// on every call: the lookup is cheap and allocates nothing, and a cached
// address would go stale if the caller reset the device or switched
// contexts between calls.
tm_status scratch_address(unsigned char** out) {
  void* p = nullptr;
  tm_status st = tmk::check_cuda(cudaGetSymbolAddress(&p, g_tm_scratch));
  if (st != TM_OK) return st;
  *out = static_cast<unsigned char*>(p);
  return TM_OK;
}

int64_t align256(int64_t x) { return (x + 255) & ~static_cast<int64_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The checks tm_quantize_qk, tm_build_mask and tm_attn_fwd make on these
// arguments, made here before anything is launched, so that a rejected call
// leaves the scratch array and the output untouched.
tm_status check_fp16(const tm_tensor* t, int64_t d) {
  if (t == nullptr || t->data == nullptr || !aligned16(t->data)) return TM_ERR_INVALID_ARG;
  if (t->T < 0 || t->H <= 0 || t->d != d) return TM_ERR_INVALID_ARG;
  if (t->stride_h < d || (t->stride_h % 8) || (t->stride_t % 8)) return TM_ERR_INVALID_ARG;
  if (t->stride_t < t->stride_h * (t->H - 1) + d) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

tm_status validate(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, const tm_tensor* out,
                   int32_t tile_m, int32_t tile_n, int32_t g, double p) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return TM_ERR_INVALID_ARG;
  if ((tile_m != 64 && tile_m != 128) || (tile_n != 64 && tile_n != 128)) return TM_ERR_UNSUPPORTED;
  if (g < 1 || !(p >= 0.0 && p <= 1.0)) return TM_ERR_INVALID_ARG;
  const int64_t D = q->d;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  const tm_tensor* ts[4] = {q, k, v, out};
  for (const tm_tensor* t : ts) {
    const tm_status st = check_fp16(t, D);
    if (st != TM_OK) return st;
  }
  if (out->T != q->T || out->H != q->H) return TM_ERR_INVALID_ARG;
  if (k->T != v->T || k->H != v->H) return TM_ERR_INVALID_ARG;
  if (q->H % k->H != 0 || q->H > 65535) return TM_ERR_INVALID_ARG;
  if (q->T > 0x7fffffffLL || k->T > 0x7fffffffLL) return TM_ERR_UNSUPPORTED;
  return TM_OK;
}

}  // namespace

extern "C" tm_status tm_attn_fwd_routed_noalloc(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v,
                                                tm_tensor* out, int32_t tile_m, int32_t tile_n, int32_t g,
                                                int32_t causal, double p, uint64_t seed, int32_t force_diag,
                                                int32_t force_sink, void* stream) {
  tm_status st = validate(q, k, v, out, tile_m, tile_n, g, p);
  if (st != TM_OK) return st;
  // Scratch layout (256-byte aligned parts): Q codes, K codes, Q scales,
  // K scales, routing mask.  The sizes come from validated shapes.
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
  st = scratch_address(&base);
  if (st != TM_OK) return st;
  int8_t* qc = reinterpret_cast<int8_t*>(base + off_qc);
  int8_t* kc = reinterpret_cast<int8_t*>(base + off_kc);
  float* qs = reinterpret_cast<float*>(base + off_qs);
  float* ks = reinterpret_cast<float*>(base + off_ks);
  uint32_t* mask = reinterpret_cast<uint32_t*>(base + off_m);

  // The INT8 fields of q, k and v are the library's here: q and k get the
  // scratch codes and scales, and v is read as plain fp16 values.
  tm_tensor qq = *q, kk = *k, vv = *v;
  qq.codes = qc;
  qq.scales = qs;
  qq.scale_kind = TM_SCALE_TILE;
  kk.codes = kc;
  kk.scales = ks;
  kk.scale_kind = TM_SCALE_TILE;
  vv.codes = nullptr;
  vv.scales = nullptr;
  vv.scale_kind = TM_SCALE_NONE;

  // Every byte read later is written first (all tiles of Q and K, every mask
  // word of every query-tile row), so nothing needs clearing between calls.
  st = tm_quantize_qk(&qq, &kk, qc, qs, kc, ks, nullptr, 0, 0, tile_m, tile_n, stream);
  if (st != TM_OK) return st;
  st = tm_build_mask(mask, static_cast<int32_t>(q->H), nullptr, 0, 0, q->T, k->T, tile_m, tile_n, g, causal, p,
                     seed, force_diag, force_sink, nqt * W, stream);
  if (st != TM_OK) return st;
  return tm_attn_fwd(&qq, &kk, &vv, out, nullptr, 0, 0, mask, nqt * W, tile_m, tile_n, g, causal, stream);
}
