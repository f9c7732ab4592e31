// tm_quant.cu -- per-tile symmetric INT8 quantisation of Q and K
// (tm_quantize_qk), and the FP8 E4M3 codes of the third precision
// (tm_quantize_qk_fp8).
//
// TileMix (Lattice paper page), abstract: the INT8 route computes score tiles
// from INT8 operands.  Rule implemented here, per (head, tile of `tile` rows of
// one sequence):  amax = max|x|;  s = fl32(amax / 127);
// code = clamp(rne(fl32(x / s)), -127, 127);  s == 0 gives codes 0.
//
// One CTA per (tile, sequence, head), Q and K in one launch: the tile's rows x
// d fp16 values arrive in shared memory by one TMA copy and stay there
// between the absmax pass and the quantise pass, so HBM traffic is one read
// of x plus one write of the codes (bytes per element: 2 read + 1 written).
// The scale is the IEEE round-to-nearest __fdiv_rn of amax by 127.  A code is
// formed from x times the correctly rounded reciprocal of the scale, rounded
// by the packed fp32 add of 1.5 * 2^23, with an exact guard: only a vector
// holding a product within 2^-15 of a half-integer takes the IEEE division,
// so the codes are bit-identical to the definition (see int8_code and
// int8_codes8).
//
// FP8 (the third precision; per-axis fp8 scales: "Add rowwise scaling to
// Float8Inference module" page, Summary): s = fl32(amax / 448), 448 being the
// largest finite E4M3 value; code = E4M3 round-to-nearest-even of
// fl32(x / s) saturating at +-448, by the hardware conversion
// cvt.rn.satfinite.e4m3x2.f32; s == 0 gives codes 0.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tm_device.cuh"
#include "tm_host.h"

namespace tmk {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantCtasPerSm = 6;

// two fp32 values to two E4M3 codes (lo in bits 0-7, hi in bits 8-15)
__device__ __forceinline__ uint32_t e4m3x2_rn_sat(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// INT8 code of x for a tile scale s > 0 with r = 1/s correctly rounded:
// rne(fl32(x / s)) clamped to [-127, 127], without a division per element.
// v = fl32(x * r) differs from x / s by at most |x / s| * 2^-23 (< 2^-16 for
// |x / s| <= 127.00002, which |x| <= amax guarantees), and fl32(x / s) by at
// most half an ulp (< 2^-17), so both lie within 2^-15 of x / s.  When v is
// farther than 2^-15 from the nearest half-integer, no rounding boundary lies
// between them and rne(v) is the code; otherwise (a near tie, about one
// element in 10^4) the IEEE division decides.
__device__ __forceinline__ int int8_code(float x, float s, float r) {
  const float v = __fmul_rn(x, r);
  float n = rintf(v);
  if (fabsf(v - n) > 0.5f - 0x1p-15f) n = rintf(__fdiv_rn(x, s));
  return max(-127, min(127, static_cast<int>(n)));
}

// One operand (Q or K) of a quantisation launch.
struct QuantOperand {
  const __half* x;
  int64_t stride_t, stride_h;
  int H;
  uint8_t* codes;
  float* scales;
  const int32_t* cu;
  int64_t L;
  int tile;
  int ntile;   // tiles per sequence launched (grid.x covers the larger operand)
  int nb;      // sequences
};

// INT8 codes of 8 fp16 values (one 16-byte vector) for a tile scale s > 0
// with r = 1/s correctly rounded, packed little-endian into two words.  Pairs
// of values go through the packed fp32 pipe: v = fl32(x * r); rne(v) by
// adding and subtracting 1.5 * 2^23 (exact for |v| < 2^22, so the sum's low
// byte is the two's-complement code and no float-to-int conversion runs);
// the same near-tie guard as int8_code, taken per vector when any of its
// eight values is within 2^-15 of a half-integer.
__device__ __forceinline__ void int8_codes8(const __half2* hv, float s, float r, uint32_t& w0, uint32_t& w1) {
  const uint64_t r2 = f2pack(r, r);
  const uint64_t mg = f2pack(12582912.0f, 12582912.0f), nmg = f2pack(-12582912.0f, -12582912.0f);
  const uint64_t neg1 = f2pack(-1.0f, -1.0f);
  uint32_t tb[8];
  float dmax = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(hv[e]);
    const uint64_t v2 = f2mul(f2pack(f.x, f.y), r2);
    const uint64_t t2 = f2add(v2, mg);
    const uint64_t n2 = f2add(t2, nmg);
    // v - n for both lanes in one packed FMA (exact: |v - n| <= 1/2 and
    // both are multiples of ulp(v), so the single rounding changes nothing)
    const uint64_t d2 = f2fma(n2, neg1, v2);
    float d0, d1, t0, t1;
    f2unpack(d2, d0, d1);
    f2unpack(t2, t0, t1);
    dmax = fmax3(dmax, fabsf(d0), fabsf(d1));
    tb[2 * e] = __float_as_uint(t0);
    tb[2 * e + 1] = __float_as_uint(t1);
  }
  if (dmax > 0.5f - 0x1p-15f) {   // a near tie: the IEEE division decides every value of the vector
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = (e & 1) ? __high2float(hv[e >> 1]) : __low2float(hv[e >> 1]);
      tb[e] = static_cast<uint32_t>(int8_code(x, s, r));
    }
  }
  w0 = __byte_perm(__byte_perm(tb[0], tb[1], 0x0040), __byte_perm(tb[2], tb[3], 0x0040), 0x5410);
  w1 = __byte_perm(__byte_perm(tb[4], tb[5], 0x0040), __byte_perm(tb[6], tb[7], 0x0040), 0x5410);
}

// One CTA per (head, tile, sequence) of either operand: grid.x runs over the
// heads of operand 0 and then those of operand 1 (heads fastest, so that the
// CTAs running at once read and write whole token rows of Q and K, all heads
// side by side).  One thread brings the tile's rows x d fp16 values into
// shared memory with a single TMA copy (rows past the tensor's end arrive as
// zeros and are not used); the absmax pass and the quantise pass then read
// them from there, so HBM traffic is one read of x plus one write of the
// codes.  With the tile in shared memory rather than in registers, six CTAs
// fit on an SM, and their copies keep 192 KB per SM in flight.
template <int D, bool F8>
__global__ void __launch_bounds__(kQuantThreads, kQuantCtasPerSm)
    quantize_tiles_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                          const QuantOperand op0, const QuantOperand op1, DevErr err) {
  constexpr int VPR = D / 8;                       // 16-byte vectors per row
  constexpr int MAXV = 128 * VPR / kQuantThreads;  // vectors per thread at tile = 128
  extern __shared__ uint8_t quant_smem_raw[];   // tile rows x D fp16, row-major, from a 128-byte boundary
  __shared__ float red[kQuantThreads / 32];
  __shared__ __align__(8) uint64_t full_bar;
  uint8_t* tile_smem = quant_smem_raw + ((128u - (smem_u32(quant_smem_raw) & 127u)) & 127u);

  const bool second = static_cast<int>(blockIdx.x) >= op0.H;
  const QuantOperand& o = second ? op1 : op0;
  const int I = blockIdx.y, b = blockIdx.z, h = second ? blockIdx.x - op0.H : blockIdx.x;
  if (I >= o.ntile || b >= o.nb) return;
  // every thread reads the same offsets (broadcast loads)
  const SeqInfo sq = seq_info(o.cu, b, o.L, o.tile);
  if (threadIdx.x == 0 && o.cu != nullptr && I == 0 && sq.len > static_cast<int64_t>(o.ntile) * o.tile)
    dev_error(err, TM_DEVERR_SEQLEN);
  const int64_t r0 = static_cast<int64_t>(I) * o.tile;
  if (r0 >= sq.len) return;
  const int rows = static_cast<int>(min(static_cast<int64_t>(o.tile), sq.len - r0));
  const int nvec = rows * VPR;
  const uint32_t bar = smem_u32(&full_bar);
  const uint32_t dst = smem_u32(tile_smem);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(o.tile) * D * 2);
    tma_load_3d(dst, second ? &tm1 : &tm0, bar, 0, h, static_cast<int32_t>(sq.start + r0));
  }
  __syncthreads();   // the barrier is initialised before any thread waits on it
  volatile int never = 0;
  mbar_wait_warp(bar, 0, err, &never);

  __half2 m2 = __float2half2_rn(0.f);
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int idx = threadIdx.x + k * kQuantThreads;
    if (idx < nvec) {
      const uint4 v = *reinterpret_cast<const uint4*>(tile_smem + idx * 16);
      const __half2* hv = reinterpret_cast<const __half2*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) m2 = __hmax2(m2, __habs2(hv[e]));
    }
  }
  float m = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  // every thread forms the tile's scale from the warp maxima (one barrier)
  float a = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) a = fmaxf(a, red[w]);
  const float sc = __fdiv_rn(a, F8 ? 448.0f : 127.0f);
  if (threadIdx.x == 0) o.scales[(sq.tile_base + I) * o.H + h] = sc;
  const float rc = sc != 0.f ? __frcp_rn(sc) : 0.f;
  const int64_t code_row_stride = static_cast<int64_t>(o.H) * D;
#pragma unroll
  for (int k = 0; k < MAXV; ++k) {
    const int idx = threadIdx.x + k * kQuantThreads;
    if (idx < nvec) {
      const int row = idx / VPR, c = idx % VPR;
      const uint4 v = *reinterpret_cast<const uint4*>(tile_smem + idx * 16);
      const __half2* hv = reinterpret_cast<const __half2*>(&v);
      uint32_t packed[2] = {0u, 0u};
      if (sc != 0.f) {
        if (F8) {
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const uint32_t pr = e4m3x2_rn_sat(__fdiv_rn(__low2float(hv[e >> 1]), sc),
                                              __fdiv_rn(__high2float(hv[e >> 1]), sc));
            packed[e >> 2] |= pr << (8 * (e & 3));
          }
        } else {
          int8_codes8(hv, sc, rc, packed[0], packed[1]);
        }
      }
      uint8_t* dst_codes = o.codes + (sq.start + r0 + row) * code_row_stride + static_cast<int64_t>(h) * D + c * 8;
      *reinterpret_cast<uint2*>(dst_codes) = make_uint2(packed[0], packed[1]);
    }
  }
}

// Asks once for the largest shared-memory carveout, so that kQuantCtasPerSm
// CTAs with their staged tiles fit on an SM (a hint; the launch is correct
// with any carveout).
std::once_flag g_quant_attr_once;
tm_status g_quant_attr_status = TM_OK;
tm_status prepare_quant_kernels() {
  std::call_once(g_quant_attr_once, [] {
    const int carve = cudaSharedmemCarveoutMaxShared;
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_tiles_kernel<128, false>, cudaFuncAttributePreferredSharedMemoryCarveout, carve);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_tiles_kernel<128, true>, cudaFuncAttributePreferredSharedMemoryCarveout, carve);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_tiles_kernel<64, false>, cudaFuncAttributePreferredSharedMemoryCarveout, carve);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(quantize_tiles_kernel<64, true>, cudaFuncAttributePreferredSharedMemoryCarveout, carve);
    g_quant_attr_status = check_cuda(e);
  });
  return g_quant_attr_status;
}

tm_status check_operand(const tm_tensor* t) {
  if (t == nullptr || t->data == nullptr) return TM_ERR_INVALID_ARG;
  if (t->T < 0 || t->H <= 0 || t->d <= 0) return TM_ERR_INVALID_ARG;
  if (t->d != 64 && t->d != 128) return TM_ERR_UNSUPPORTED;
  if (t->stride_h < t->d || t->stride_t < t->stride_h * (t->H - 1) + t->d) return TM_ERR_INVALID_ARG;
  if ((t->stride_h % 8) || (t->stride_t % 8)) return TM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->data) % 16) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

// Checks one operand's outputs and fills its launch description; *empty is
// set when it has nothing to quantise.
tm_status make_operand(const tm_tensor* x, void* codes_ptr, float* scales, const int32_t* cu, int32_t batch,
                       int32_t max_seqlen, int32_t tile, QuantOperand* o, bool* empty) {
  uint8_t* codes = static_cast<uint8_t*>(codes_ptr);
  if (codes == nullptr || scales == nullptr) return TM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(codes) % 16 || reinterpret_cast<uintptr_t>(scales) % 4)
    return TM_ERR_INVALID_ARG;
  const int64_t maxlen = cu ? max_seqlen : x->T;
  const int nb = cu ? batch : 1;
  *empty = maxlen <= 0 || nb <= 0;
  if (*empty) return TM_OK;
  const int64_t ntile = (maxlen + tile - 1) / tile;
  if (ntile > 0x7fffffff || nb > 65535 || x->H > 65535) return TM_ERR_UNSUPPORTED;
  o->x = static_cast<const __half*>(x->data);
  o->stride_t = x->stride_t;
  o->stride_h = x->stride_h;
  o->H = static_cast<int>(x->H);
  o->codes = codes;
  o->scales = scales;
  o->cu = cu;
  o->L = x->T;
  o->tile = tile;
  o->ntile = static_cast<int>(ntile);
  o->nb = nb;
  return TM_OK;
}

// Quantises x (and y, when given) in one launch.
tm_status launch_quant(const tm_tensor* x, void* x_codes, float* x_scales, const int32_t* cu_x, int32_t max_x,
                       int32_t tile_x, const tm_tensor* y, void* y_codes, float* y_scales, const int32_t* cu_y,
                       int32_t max_y, int32_t tile_y, int32_t batch, cudaStream_t stream, bool f8) {
  QuantOperand o[2] = {};
  bool empty[2] = {true, true};
  tm_status st = make_operand(x, x_codes, x_scales, cu_x, batch, max_x, tile_x, &o[0], &empty[0]);
  if (st != TM_OK) return st;
  if (y != nullptr) {
    st = make_operand(y, y_codes, y_scales, cu_y, batch, max_y, tile_y, &o[1], &empty[1]);
    if (st != TM_OK) return st;
  }
  // an empty operand takes no heads of the grid
  if (empty[0]) o[0].H = 0;
  if (empty[1]) o[1].H = 0;
  const int64_t heads = static_cast<int64_t>(o[0].H) + o[1].H;
  if (heads == 0) return TM_OK;
  if (heads > 65535) return TM_ERR_UNSUPPORTED;
  const int gx = max(empty[0] ? 0 : o[0].ntile, empty[1] ? 0 : o[1].ntile);
  const int gy = max(empty[0] ? 0 : o[0].nb, empty[1] ? 0 : o[1].nb);
  if (gx > 65535) return TM_ERR_UNSUPPORTED;   // tiles per sequence on grid.y
  dim3 grid(static_cast<unsigned>(heads), static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  DevErr err{device_error_word()};
  const int64_t d = x->d;
  // one TMA map per operand: box of one tile (tile rows x d), no swizzle
  CUtensorMap map[2];
  const tm_tensor* src[2] = {x, y};
  for (int i = 0; i < 2; ++i) {
    if (empty[i]) continue;
    st = encode_thd_map(&map[i], src[i]->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, src[i]->T, src[i]->H, d,
                        src[i]->stride_t, src[i]->stride_h, static_cast<int>(d), o[i].tile,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != TM_OK) return st;
  }
  if (empty[0]) map[0] = map[1];
  if (empty[1]) map[1] = map[0];
  // the larger operand tile, plus room to align it to 128 bytes (TMA destination)
  const size_t smem = static_cast<size_t>(max(empty[0] ? 0 : o[0].tile, empty[1] ? 0 : o[1].tile)) * d * 2 + 128;
  st = prepare_quant_kernels();
  if (st != TM_OK) return st;
  if (d == 128 && f8)
    quantize_tiles_kernel<128, true><<<grid, kQuantThreads, smem, stream>>>(map[0], map[1], o[0], o[1], err);
  else if (d == 128)
    quantize_tiles_kernel<128, false><<<grid, kQuantThreads, smem, stream>>>(map[0], map[1], o[0], o[1], err);
  else if (f8)
    quantize_tiles_kernel<64, true><<<grid, kQuantThreads, smem, stream>>>(map[0], map[1], o[0], o[1], err);
  else
    quantize_tiles_kernel<64, false><<<grid, kQuantThreads, smem, stream>>>(map[0], map[1], o[0], o[1], err);
  return check_cuda(cudaGetLastError());
}

}  // namespace
}  // namespace tmk

extern "C" tm_status tm_quantize_qk_varlen(const tm_tensor* q, const tm_tensor* k, int8_t* q_codes,
                                           float* q_scales, int8_t* k_codes, float* k_scales,
                                           const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                           int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                           int32_t tile_m, int32_t tile_n, void* stream) {
  using namespace tmk;
  if ((tile_m != 64 && tile_m != 128) || (tile_n != 64 && tile_n != 128)) return TM_ERR_UNSUPPORTED;
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr || batch <= 0 || max_seqlen_q <= 0) return TM_ERR_INVALID_ARG;
  tm_status st = check_operand(q);
  if (st != TM_OK) return st;
  if (k != nullptr) {
    st = check_operand(k);
    if (st != TM_OK) return st;
    if (k->d != q->d || max_seqlen_k <= 0) return TM_ERR_INVALID_ARG;
  }
  return launch_quant(q, q_codes, q_scales, cu_seqlens_q, max_seqlen_q, tile_m, k, k_codes, k_scales, cu_seqlens_k,
                      max_seqlen_k, tile_n, batch, as_stream(stream), false);
}

extern "C" tm_status tm_quantize_qk(const tm_tensor* q, const tm_tensor* k, int8_t* q_codes,
                                    float* q_scales, int8_t* k_codes, float* k_scales,
                                    const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen,
                                    int32_t tile_m, int32_t tile_n, void* stream) {
  using namespace tmk;
  if ((tile_m != 64 && tile_m != 128) || (tile_n != 64 && tile_n != 128)) return TM_ERR_UNSUPPORTED;
  tm_status st = check_operand(q);
  if (st != TM_OK) return st;
  if (k != nullptr) {
    st = check_operand(k);
    if (st != TM_OK) return st;
    if (k->d != q->d) return TM_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && k->T != q->T) return TM_ERR_INVALID_ARG;
  }
  if (cu_seqlens != nullptr && (batch <= 0 || max_seqlen <= 0)) return TM_ERR_INVALID_ARG;
  return launch_quant(q, q_codes, q_scales, cu_seqlens, max_seqlen, tile_m, k, k_codes, k_scales, cu_seqlens,
                      max_seqlen, tile_n, batch, as_stream(stream), false);
}

extern "C" tm_status tm_quantize_qk_fp8(const tm_tensor* q, const tm_tensor* k, uint8_t* q_codes, float* q_scales,
                                        uint8_t* k_codes, float* k_scales, const int32_t* cu_seqlens, int32_t batch,
                                        int32_t max_seqlen, int32_t tile_m, int32_t tile_n, void* stream) {
  using namespace tmk;
  if ((tile_m != 64 && tile_m != 128) || (tile_n != 64 && tile_n != 128)) return TM_ERR_UNSUPPORTED;
  tm_status st = check_operand(q);
  if (st != TM_OK) return st;
  if (k != nullptr) {
    st = check_operand(k);
    if (st != TM_OK) return st;
    if (k->d != q->d) return TM_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && k->T != q->T) return TM_ERR_INVALID_ARG;
  }
  if (cu_seqlens != nullptr && (batch <= 0 || max_seqlen <= 0)) return TM_ERR_INVALID_ARG;
  return launch_quant(q, q_codes, q_scales, cu_seqlens, max_seqlen, tile_m, k, k_codes, k_scales, cu_seqlens,
                      max_seqlen, tile_n, batch, as_stream(stream), true);
}
