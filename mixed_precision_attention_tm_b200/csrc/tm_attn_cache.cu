// tm_attn_cache.cu -- fused tile-routed attention over an INT8 K/V cache.
//
// TileMix (Lattice paper page), abstract: tile-routed FP16/INT8 attention
// supports INT8 key/value caches.  The cache stores int8 codes with one fp16
// scale per (token, KV head); its fp16 view is fp16_rn(code * scale).
//   * INT8-routed key groups multiply the int8 Q tile codes with the cached
//     int8 K codes directly (tcgen05.mma kind::i8); the softmax applies
//     s_q * s_k[j] * sigma per key column j.
//   * FP16-routed key groups and all of V use the fp16 view, produced in
//     shared memory by a dequantisation warpgroup from TMA-loaded code tiles
//     (written in the 128-byte-swizzled layout the tensor core reads).
//
// One CTA owns one query tile (tile_m = 64 or 128 rows; 128-row MMA), key
// tiles of 128, d = 128.  Warps: 0-3 softmax (one row per thread, TMEM lane =
// row), 4-7 dequantisation (one key row per thread), 8 TMA producer, 9
// tcgen05 issuer, 10-11 idle.  TMEM: S double-buffered (P overwrites S as
// fp16), O fp32.  Every mbarrier wait is bounded (tm_device.cuh).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tm_attn_internal.h"
#include "tm_device.cuh"
#include "tm_host.h"


// Phase profile (compiled only with TM_PHASES and TM_TRACE): thread 0 (softmax)
// and thread 128 (dequantisation) of the traced CTA sum SM-clock deltas per
// phase in registers and store the sums once.
#if defined(TM_PHASES) && defined(TM_TRACE)
#define TMC_PH_DECL long long tm_ph[8] = {0, 0, 0, 0, 0, 0, 0, 0}; long long tm_ph_t = clock64();
#define TMC_PH(i) do { const long long tm_now = clock64(); tm_ph[i] += tm_now - tm_ph_t; tm_ph_t = tm_now; } while (0)
#define TMC_PH_STORE(role) do { if ((threadIdx.x & 127) == 0 && blockIdx.x == g_tm_trace_block) \
  for (int i = 0; i < 8; ++i) g_tm_trace[role][TM_TRACE_EVENTS - 8 + i] = static_cast<unsigned long long>(tm_ph[i]); } while (0)
#else
#define TMC_PH_DECL
#define TMC_PH(i) do { } while (0)
#define TMC_PH_STORE(role) do { } while (0)
#endif

#ifdef TM_TRACE
// Trace-build reader of this translation unit's trace buffer (same contract
// as tm_debug_trace_read for the pair kernel).
extern "C" int tm_debug_trace_read_cache(unsigned long long* host, unsigned int block) {
  if (host == nullptr) {
    static unsigned long long zero[TM_TRACE_ROLES][TM_TRACE_EVENTS];
    if (cudaMemcpyToSymbol(g_tm_trace, zero, sizeof(zero)) != cudaSuccess) return -1;
    return cudaMemcpyToSymbol(g_tm_trace_block, &block, sizeof(block)) == cudaSuccess ? 0 : -1;
  }
  return cudaMemcpyFromSymbol(host, g_tm_trace, sizeof(g_tm_trace)) == cudaSuccess ? 0 : -1;
}
#endif

namespace tmk {
namespace {

struct CfgC {
  static constexpr int D = 128, BM = 128, BN = 128;
  static constexpr int Q16_BYTES = BM * D * 2;       // 32 KB
  static constexpr int Q8_BYTES = BM * D;            // 16 KB
  static constexpr int C8 = BN * D;                  // one int8 code tile, 16 KB
  static constexpr int F16 = BN * D * 2;             // one fp16 tile, 32 KB
  static constexpr int HALF = BN * 128;              // 64-column fp16 slab
  static constexpr int NKC = 2, NK16 = 1, NVC = 2, NV16 = 2;
  static constexpr int OFF_Q16 = 0;
  static constexpr int OFF_Q8 = OFF_Q16 + Q16_BYTES;
  static constexpr int OFF_KC = OFF_Q8 + Q8_BYTES;
  static constexpr int OFF_K16 = OFF_KC + NKC * C8;
  static constexpr int OFF_VC = OFF_K16 + NK16 * F16;
  static constexpr int OFF_V16 = OFF_VC + NVC * C8;
  static constexpr int OFF_BAR = OFF_V16 + NV16 * F16;
  static constexpr int BAR_BYTES = 1024;             // barriers + key-scale staging (512 B)
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL = 2 * BN;
  static constexpr uint32_t IDESC_S16 = idesc_f16(BM, BN, false);
  static constexpr uint32_t IDESC_S8 = idesc_i8(BM, BN);
  static constexpr uint32_t IDESC_PV = idesc_f16(BM, D, true);
  static constexpr int THREADS = 384;
  // launch: 168 registers per thread (3 warps per SM sub-partition); softmax
  // takes 232, the control warpgroup gives back to 104, dequantisation keeps
  // 168: 128 * (232 + 168 + 104) = 384 * 168.
  static constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 232, CONTROL_REGS = 104;
  static_assert(128 * (SOFTMAX_REGS + LAUNCH_REGS + CONTROL_REGS) == THREADS * LAUNCH_REGS, "register split");
};

enum {
  K_QFULL = 0,
  K_KCFULL = 1,    // +NKC
  K_KCEMPTY = 3,   // +NKC (count 129: dequant threads + issuer commit)
  K_K16FULL = 5,   // +NK16 (count 128)
  K_K16EMPTY = 6,  // +NK16
  K_VCFULL = 7,    // +NVC
  K_VCEMPTY = 9,   // +NVC (count 128)
  K_V16FULL = 11,  // +NV16 (count 128)
  K_V16EMPTY = 13, // +NV16
  K_SFULL = 15,    // +2
  K_PFULL = 17,    // +2 (count 128)
  K_ODONE = 19,
  K_DRAIN = 20,
  K_COUNT = 21
};

struct ParamsC {
  __half* out;
  int64_t out_st, out_sh;
  const float* q_scales;        // [n_qtiles, Hq]
  const __half* k_tok_scale;    // [T, Hkv]
  const __half* v_tok_scale;    // [T, Hkv]
  const uint32_t* bitmask;
  int64_t mask_hs;
  int W;
  const int32_t* cu;
  const int32_t* cu_k;   // key offsets (= cu unless separate)
  int64_t max_lk;        // longest key row the launch was sized for
  int64_t Lq, Lk;
  int Hq, Hkv, tile_m, g, causal, n_qt_max, batch;
  float scale_log2;
  DevErr err;
};

// exp2 pairs (of every 8) the softmax evaluates on the FMA pipe instead of MUFU
#ifndef TM_CACHE_EXP2_EMU_PAIRS
#define TM_CACHE_EXP2_EMU_PAIRS 3
#endif
constexpr int kCacheEmuPairs = TM_CACHE_EXP2_EMU_PAIRS;

__device__ __forceinline__ bool route_c(const uint32_t* row, int g, int j) {
  if (row == nullptr) return false;
  const int G = j / g;
  return (__ldg(row + (G >> 5)) >> (G & 31)) & 1u;
}

// Row r of a 128-byte-swizzled int8 code tile (128 codes) -> the same row of a
// 128-byte-swizzled fp16 tile (two 64-column slabs), each value
// fp16_rn(code * scale).  Codes become fp16 without integer-to-float
// conversions: XOR 0x80 turns a code x into the byte x + 128, which placed
// under the fp16 exponent byte 0x64 reads as 1024 + x + 128 exactly (ulp 1);
// subtracting 1152 gives x exactly, and one fp16 multiply by the (fp16)
// scale rounds the exact product once, as fp16_rn(x * scale) requires.
__device__ __forceinline__ void dequant_row(const uint8_t* codes, uint8_t* f16, int r, __half scale) {
  const int sw = r & 7;
  const __half2 bias = __float2half2_rn(1152.0f);
  const __half2 s2 = __half2half2(scale);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 raw = *reinterpret_cast<const uint4*>(codes + r * 128 + ((c ^ sw) << 4));
    const uint32_t w[4] = {raw.x ^ 0x80808080u, raw.y ^ 0x80808080u, raw.z ^ 0x80808080u, raw.w ^ 0x80808080u};
    uint32_t h[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t lo = __byte_perm(w[q], 0x64646464u, 0x4140u);   // bytes b0, 0x64, b1, 0x64
      uint32_t hi = __byte_perm(w[q], 0x64646464u, 0x4342u);   // bytes b2, 0x64, b3, 0x64
      __half2 vlo = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&lo), bias), s2);
      __half2 vhi = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&hi), bias), s2);
      h[2 * q] = *reinterpret_cast<uint32_t*>(&vlo);
      h[2 * q + 1] = *reinterpret_cast<uint32_t*>(&vhi);
    }
    // codes 16c..16c+15 = fp16 columns 16c..16c+15: slab c/4, chunks 2(c%4), 2(c%4)+1
    uint8_t* slab = f16 + (c >> 2) * CfgC::HALF + r * 128;
    const int c0 = 2 * (c & 3);
    *reinterpret_cast<uint4*>(slab + ((c0 ^ sw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(slab + (((c0 + 1) ^ sw) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

__global__ void __launch_bounds__(384, 1)
    attn_cache_kernel(const __grid_constant__ CUtensorMap tmQ16, const __grid_constant__ CUtensorMap tmQ8,
                      const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                      const ParamsC p) {
  using C = CfgC;
  constexpr int BN = C::BN, D = C::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * K_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * K_COUNT + 4);
  float* kscale_s = reinterpret_cast<float*>(smem + C::OFF_BAR + 512);   // [128], softmax-private

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int h = blockIdx.x % p.Hq;
  const int t1 = blockIdx.x / p.Hq;
  const int b = t1 % p.batch;
  const int I = p.n_qt_max - 1 - t1 / p.batch;
  const SeqInfo sq = seq_info(p.cu, b, p.Lq, p.tile_m);
  const int64_t Lq = sq.len;
  // keys of sequence b: rows cu_k[b] .. (cu_k = cu unless the key offsets
  // differ, as in prefix-cached prefill); a longer key row than the launch
  // was sized for (mask words, key scales) is an argument error
  const SeqInfo skq = seq_info(p.cu_k, b, p.Lk, BN);
  const int64_t Lk = p.cu_k ? skq.len : p.Lk;
  const int64_t kstart = p.cu_k ? skq.start : 0;
  if (p.cu_k != nullptr && Lk > p.max_lk) {
    if (threadIdx.x == 0) dev_error(p.err, TM_DEVERR_SEQLEN);
    return;
  }
  if (p.cu != nullptr && I == 0 && threadIdx.x == 0 && Lq > static_cast<int64_t>(p.n_qt_max) * p.tile_m)
    dev_error(p.err, TM_DEVERR_SEQLEN);
  if (static_cast<int64_t>(I) * p.tile_m >= Lq) return;

  const int rows_valid = static_cast<int>(min(static_cast<int64_t>(p.tile_m), Lq - static_cast<int64_t>(I) * p.tile_m));
  int64_t jmax = Lk - 1;
  if (p.causal) jmax = min(jmax, static_cast<int64_t>(I) * p.tile_m + rows_valid - 1 + Lk - Lq);
  const int nJ = (Lk <= 0 || jmax < 0) ? 0 : static_cast<int>(jmax / BN + 1);
  const int64_t ig = sq.tile_base + I;
  const int hk = h / (p.Hq / p.Hkv);
  const uint32_t* mrow = p.bitmask ? p.bitmask + static_cast<int64_t>(h) * p.mask_hs + ig * p.W : nullptr;
  const int64_t qrow0 = sq.start + static_cast<int64_t>(I) * p.tile_m;

  if (threadIdx.x == 0) {
    mbar_init(bar(K_QFULL), 1);
    for (int s = 0; s < C::NKC; ++s) { mbar_init(bar(K_KCFULL + s), 1); mbar_init(bar(K_KCEMPTY + s), 129); }
    for (int s = 0; s < C::NK16; ++s) { mbar_init(bar(K_K16FULL + s), 128); mbar_init(bar(K_K16EMPTY + s), 1); }
    for (int s = 0; s < C::NVC; ++s) { mbar_init(bar(K_VCFULL + s), 1); mbar_init(bar(K_VCEMPTY + s), 128); }
    for (int s = 0; s < C::NV16; ++s) { mbar_init(bar(K_V16FULL + s), 128); mbar_init(bar(K_V16EMPTY + s), 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(bar(K_SFULL + s), 1); mbar_init(bar(K_PFULL + s), 128); }
    mbar_init(bar(K_ODONE), 1);
    mbar_init(bar(K_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_dec<C::CONTROL_REGS>();
    if (warp == 8 && lane == 0 && nJ > 0) {
      // ======================= TMA producer =======================
      bool any8 = false;
      if (mrow != nullptr)
        for (int w = 0; w < p.W; ++w) any8 |= (__ldg(mrow + w) != 0u);
      mbar_arrive_expect_tx(bar(K_QFULL), C::Q16_BYTES + (any8 ? C::Q8_BYTES : 0));
      tma_load_3d(sbase + C::OFF_Q16, &tmQ16, bar(K_QFULL), 0, h, static_cast<int32_t>(qrow0));
      tma_load_3d(sbase + C::OFF_Q16 + C::HALF, &tmQ16, bar(K_QFULL), 64, h, static_cast<int32_t>(qrow0));
      if (any8) tma_load_3d(sbase + C::OFF_Q8, &tmQ8, bar(K_QFULL), 0, h, static_cast<int32_t>(qrow0));
      int nkc = 0, nvc = 0;
      for (int j = 0; j < nJ; ++j) {
        const int32_t krow = static_cast<int32_t>(kstart + static_cast<int64_t>(j) * BN);
        const int s = j % C::NKC, lap = j / C::NKC;
        if (lap > 0 && !mbar_wait(bar(K_KCEMPTY + s), (lap - 1) & 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(bar(K_KCFULL + s), C::C8);
        tma_load_3d(sbase + C::OFF_KC + s * C::C8, &tmKc, bar(K_KCFULL + s), 0, hk, krow);
        ++nkc;
        const int vs = j % C::NVC, vlap = j / C::NVC;
        if (vlap > 0 && !mbar_wait(bar(K_VCEMPTY + vs), (vlap - 1) & 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(bar(K_VCFULL + vs), C::C8);
        tma_load_3d(sbase + C::OFF_VC + vs * C::C8, &tmVc, bar(K_VCFULL + vs), 0, hk, krow);
        ++nvc;
      }
      volatile int never = 0;
      mbar_wait(bar(K_QFULL), 0, p.err, &never);
      for (int s = 0; s < C::NKC; ++s) {
        const int cnt = nkc > s ? (nkc - 1 - s) / C::NKC + 1 : 0;
        if (cnt > 0) mbar_wait(bar(K_KCFULL + s), (cnt - 1) & 1, p.err, &never);
      }
      for (int s = 0; s < C::NVC; ++s) {
        const int cnt = nvc > s ? (nvc - 1 - s) / C::NVC + 1 : 0;
        if (cnt > 0) mbar_wait(bar(K_VCFULL + s), (cnt - 1) & 1, p.err, &never);
      }
    } else if (warp == 9 && nJ > 0) {
      // ======================= tcgen05 issuer =======================
      // Whole warp: descriptors are warp-uniform values built ahead of each
      // group; one elected lane issues the group and its commits.
      bool ok = mbar_wait_warp(bar(K_QFULL), 0, p.err, abort_flag);
      int n16 = 0;
      auto commit1 = [&](uint32_t b) {
        if (elect_one()) tc_commit(b);
        __syncwarp();
      };
      auto issue_pv = [&](int t) -> bool {
        const int vs = t % C::NV16;
        const uint32_t vb = sbase + C::OFF_V16 + vs * C::F16;
        uint64_t bd[BN / 16];
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) bd[kk] = smem_desc(vb + kk * 2048, C::HALF, 1024, kSwizzle128);
        if (!mbar_wait_warp(bar(K_PFULL + (t & 1)), (t >> 1) & 1, p.err, abort_flag)) return false;
        if (!mbar_wait_warp(bar(K_V16FULL + vs), (t / C::NV16) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t a_tmem = tmem + static_cast<uint32_t>(t & 1) * BN;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_f16_ts(tmem + C::O_COL, a_tmem + kk * 8, bd[kk], C::IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(K_ODONE));
          tc_commit(bar(K_V16EMPTY + vs));
        }
        __syncwarp();
        return true;
      };
      for (int j = 0; ok && j < nJ; ++j) {
        const bool i8 = route_c(mrow, p.g, j);
        const int s = j % C::NKC;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(j & 1) * BN;
        if (i8) {
          const uint32_t kb = sbase + C::OFF_KC + s * C::C8;
          uint64_t ad[D / 32], bd[D / 32];
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            ad[kk] = smem_desc(sbase + C::OFF_Q8 + kk * 32, 16, 1024, kSwizzle128);
            bd[kk] = smem_desc(kb + kk * 32, 16, 1024, kSwizzle128);
          }
          if (!(ok = mbar_wait_warp(bar(K_KCFULL + s), (j / C::NKC) & 1, p.err, abort_flag))) break;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) mma_i8_ss(d_tmem, ad[kk], bd[kk], C::IDESC_S8, kk > 0 ? 1u : 0u);
            tc_commit(bar(K_SFULL + (j & 1)));
          }
          __syncwarp();
        } else {
          const int s16 = n16 % C::NK16;
          const uint32_t kb = sbase + C::OFF_K16 + s16 * C::F16;
          uint64_t ad[D / 16], bd[D / 16];
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::HALF + (kk & 3) * 32;
            ad[kk] = smem_desc(sbase + C::OFF_Q16 + off, 16, 1024, kSwizzle128);
            bd[kk] = smem_desc(kb + off, 16, 1024, kSwizzle128);
          }
          if (!(ok = mbar_wait_warp(bar(K_K16FULL + s16), (n16 / C::NK16) & 1, p.err, abort_flag))) break;
          tc_fence_after();   // dequantised tile written by the generic proxy, fenced by its writers
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) mma_f16_ss(d_tmem, ad[kk], bd[kk], C::IDESC_S16, kk > 0 ? 1u : 0u);
            tc_commit(bar(K_SFULL + (j & 1)));
            tc_commit(bar(K_K16EMPTY + s16));
          }
          __syncwarp();
          ++n16;
        }
        commit1(bar(K_KCEMPTY + s));
        if (j >= 1 && !(ok = issue_pv(j - 1))) break;
      }
      if (ok) issue_pv(nJ - 1);
      commit1(bar(K_DRAIN));
      volatile int never = 0;
      mbar_wait_warp(bar(K_DRAIN), 0, p.err, &never);
    }
  } else if (warp >= 4) {
    // ======================= dequantisation (one key row per thread) ==========
    const int r = threadIdx.x - 128;
    int n16 = 0;
    TMC_PH_DECL
    for (int j = 0; j < nJ; ++j) {
      const bool i8 = route_c(mrow, p.g, j);
      const int64_t tok = kstart + static_cast<int64_t>(j) * BN + r;
      const bool in = tok < kstart + Lk;
      const __half ks = in ? p.k_tok_scale[tok * p.Hkv + hk] : __float2half(0.f);
      const __half vs = in ? p.v_tok_scale[tok * p.Hkv + hk] : __float2half(0.f);
      const int s = j % C::NKC;
      if (!mbar_wait(bar(K_KCFULL + s), (j / C::NKC) & 1, p.err, abort_flag)) break;
      TMC_PH(0);
      if (!i8) {
        const int s16 = n16 % C::NK16;
        if (n16 >= C::NK16 && !mbar_wait(bar(K_K16EMPTY + s16), ((n16 / C::NK16) - 1) & 1, p.err, abort_flag)) break;
        TMC_PH(1);
        dequant_row(smem + C::OFF_KC + s * C::C8, smem + C::OFF_K16 + s16 * C::F16, r, ks);
        fence_async_shared();
        mbar_arrive(bar(K_K16FULL + s16));
        ++n16;
      }
      mbar_arrive(bar(K_KCEMPTY + s));
      TMC_PH(2);
      const int vcs = j % C::NVC;
      if (!mbar_wait(bar(K_VCFULL + vcs), (j / C::NVC) & 1, p.err, abort_flag)) break;
      TMC_PH(3);
      const int v16 = j % C::NV16;
      if (j >= C::NV16 && !mbar_wait(bar(K_V16EMPTY + v16), ((j / C::NV16) - 1) & 1, p.err, abort_flag)) break;
      TMC_PH(4);
      dequant_row(smem + C::OFF_VC + vcs * C::C8, smem + C::OFF_V16 + v16 * C::F16, r, vs);
      fence_async_shared();
      mbar_arrive(bar(K_V16FULL + v16));
      mbar_arrive(bar(K_VCEMPTY + vcs));
      TMC_PH(5);
    }
    TMC_PH_STORE(1);
  } else {
    // ======================= softmax (warps 0-3) =======================
    regs_inc<C::SOFTMAX_REGS>();
    const int r = threadIdx.x;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool row_ok = r < rows_valid;
    const int64_t i_row = static_cast<int64_t>(I) * p.tile_m + r;
    int64_t lim = -1;
    if (row_ok) lim = p.causal ? min(Lk - 1, i_row + Lk - Lq) : Lk - 1;
    float c8_row = 0.f;
    if (mrow != nullptr) c8_row = __ldg(p.q_scales + ig * p.Hq + h) * p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    TMC_PH_DECL
    for (int j = 0; j < nJ; ++j) {
      const bool i8 = route_c(mrow, p.g, j);
      if (i8) {
        // per-column key scales of this tile, shared by the four softmax warps
        const int64_t tok = kstart + static_cast<int64_t>(j) * BN + r;
        const float ks = tok < kstart + Lk ? __half2float(p.k_tok_scale[tok * p.Hkv + hk]) : 0.f;
        named_bar_sync(1, 128);            // previous INT8 tile's readers are done
        kscale_s[r] = ks * c8_row;
        named_bar_sync(1, 128);
      }
      if (!mbar_wait(bar(K_SFULL + (j & 1)), (j >> 1) & 1, p.err, abort_flag)) { ok = false; break; }
      tc_fence_after();
      __syncwarp();
      TMC_PH(0);
      float x[BN];
      {
        uint32_t u[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc)
          tmem_ld32p(lane_addr + static_cast<uint32_t>(j & 1) * BN + cc * 32, u + cc * 32);
        tmem_wait_ld_regs<BN>(u);
        TMC_PH(1);
        if (i8) {
          // exact int32 -> fp32 (|acc| < 2^22: add the bits of 1.5 * 2^23, then
          // subtract it), times the column's s_q s_k sigma log2(e), in f32x2
          const uint64_t nmagic = f2pack(-12582912.0f, -12582912.0f);
          const float2* ks2 = reinterpret_cast<const float2*>(kscale_s);
#pragma unroll
          for (int e = 0; e < BN; e += 2) {
            const float2 kk = ks2[e >> 1];
            const uint64_t v = f2mul(f2add(f2pack(__int_as_float(static_cast<int>(u[e]) + 0x4B400000),
                                                  __int_as_float(static_cast<int>(u[e + 1]) + 0x4B400000)),
                                           nmagic),
                                     f2pack(kk.x, kk.y));
            f2unpack(v, x[e], x[e + 1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < BN; ++e) x[e] = __uint_as_float(u[e]);
        }
      }
      // scores in log2 units are x * c (INT8 tiles are already scaled)
      const float c = i8 ? 1.0f : p.scale_log2;
      const int64_t nv64 = lim - static_cast<int64_t>(j) * BN + 1;
      const int nv = nv64 <= 0 ? 0 : (nv64 >= BN ? BN : static_cast<int>(nv64));
      if (!__all_sync(0xffffffffu, nv == BN)) {
#pragma unroll
        for (int e = 0; e < BN; ++e) x[e] = (e < nv) ? x[e] : -INFINITY;
      }
      float alpha = 1.f;
      if (nv > 0) {
        const float mt = row_max<BN>(x) * c;
        if (mt > m_used + kLazyRescaleLog2) {
          alpha = ex2_approx(m_used - mt);
          m_used = mt;
        }
      }
      const float msub = (m_used == -INFINITY) ? 0.f : m_used;
      TMC_PH(2);
      const uint64_t c2 = f2pack(c, c);
      const uint64_t nm2 = f2pack(-msub, -msub);
      uint32_t pk[BN / 2];
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < BN; e += 2) {
        const uint64_t y2 = f2fma(f2pack(x[e], x[e + 1]), c2, nm2);
        float p0, p1;
        if (kCacheEmuPairs > 0 && ((e >> 1) & 7) < kCacheEmuPairs) {
          exp2_poly2(y2, p0, p1);
        } else {
          float y0, y1;
          f2unpack(y2, y0, y1);
          p0 = ex2_approx(y0);
          p1 = ex2_approx(y1);
        }
        acc2[(e >> 1) & 3] = f2add(acc2[(e >> 1) & 3], f2pack(p0, p1));
        pk[e >> 1] = pack_half2(p0, p1);
      }
      {
        const uint64_t s2 = f2add(f2add(acc2[0], acc2[1]), f2add(acc2[2], acc2[3]));
        float s0, s1;
        f2unpack(s2, s0, s1);
        l = l * alpha + (s0 + s1);
      }
      TMC_PH(3);
      // O is rescaled only when a row of this warp raised its running max;
      // then PV_{j-1} must have completed.  S_j was committed after PV_{j-2}
      // was issued, so o_done has finished phase j-2, and PV_j cannot start
      // before this warp releases P_j: waiting for phase j-1 by parity is
      // unambiguous although earlier phases were skipped.  The last tile
      // always waits, so that the epilogue's wait for phase nJ-1 can only
      // see phase nJ-1 or nJ (parity alone cannot tell nJ-2 from nJ).
      const bool rescale = j > 0 && __any_sync(0xffffffffu, alpha != 1.f);
      if (j > 0 && (rescale || j == nJ - 1)) {
        if (!mbar_wait(bar(K_ODONE), (j - 1) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        __syncwarp();
      }
      if (rescale) {
        uint32_t o[D];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld32p(lane_addr + C::O_COL + cc * 32, o + cc * 32);
        tmem_wait_ld_regs<D>(o);
        const uint64_t a2 = f2pack(alpha, alpha);
#pragma unroll
        for (int e = 0; e < D; e += 2) {
          float o0, o1;
          f2unpack(f2mul(f2pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), o0, o1);
          o[e] = __float_as_uint(o0);
          o[e + 1] = __float_as_uint(o1);
        }
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_st32p(lane_addr + C::O_COL + cc * 32, o + cc * 32);
      }
      TMC_PH(4);
      __syncwarp();
#pragma unroll
      for (int cc = 0; cc < BN / 64; ++cc)
        tmem_st32p(lane_addr + static_cast<uint32_t>(j & 1) * BN + cc * 32, pk + cc * 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(K_PFULL + (j & 1)));
      TMC_PH(5);
    }
    TMC_PH_STORE(0);
    bool have_o = false;
    if (ok && nJ > 0) {
      have_o = mbar_wait(bar(K_ODONE), (nJ - 1) & 1, p.err, abort_flag);
      tc_fence_after();
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    __syncwarp();
    uint32_t o[D];
    if (__all_sync(0xffffffffu, have_o)) {
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32p(lane_addr + C::O_COL + cc * 32, o + cc * 32);
      tmem_wait_ld_regs<D>(o);
    } else {
#pragma unroll
      for (int e = 0; e < D; ++e) o[e] = 0u;
    }
    if (row_ok) {
      __half* orow = p.out + (sq.start + i_row) * p.out_st + static_cast<int64_t>(h) * p.out_sh;
#pragma unroll
      for (int cc = 0; cc < D / 8; ++cc) {
        uint4 pkt;
        pkt.x = pack_half2(__uint_as_float(o[8 * cc + 0]) * inv, __uint_as_float(o[8 * cc + 1]) * inv);
        pkt.y = pack_half2(__uint_as_float(o[8 * cc + 2]) * inv, __uint_as_float(o[8 * cc + 3]) * inv);
        pkt.z = pack_half2(__uint_as_float(o[8 * cc + 4]) * inv, __uint_as_float(o[8 * cc + 5]) * inv);
        pkt.w = pack_half2(__uint_as_float(o[8 * cc + 6]) * inv, __uint_as_float(o[8 * cc + 7]) * inv);
        st_global_stream_v4(reinterpret_cast<uint4*>(orow) + cc, pkt);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

std::mutex g_mu_c;

}  // namespace

tm_status launch_attn_cache(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t tile_m, int32_t g,
                            int32_t causal, cudaStream_t stream) {
  using C = CfgC;
  static bool attr_done = false;
  {
    std::lock_guard<std::mutex> lk(g_mu_c);
    if (!attr_done) {
      cudaFuncAttributes fa;
      tm_status st = check_cuda(cudaFuncGetAttributes(&fa, attn_cache_kernel));
      if (st != TM_OK) return st;
      if (fa.numRegs != C::LAUNCH_REGS) return TM_ERR_UNSUPPORTED;
      st = check_cuda(cudaFuncSetAttribute(attn_cache_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::SMEM_BYTES));
      if (st != TM_OK) return st;
      attr_done = true;
    }
  }
  CUtensorMap mQ16, mQ8, mKc, mVc;
  tm_status st;
  st = encode_thd_map(&mQ16, q->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, q->T, q->H, C::D, q->stride_t,
                      q->stride_h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mKc, k->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k->T, k->H, C::D, k->H * C::D, C::D,
                      C::D, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mVc, v->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, v->T, v->H, C::D, v->H * C::D, C::D,
                      C::D, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  if (bitmask != nullptr) {
    st = encode_thd_map(&mQ8, q->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->T, q->H, C::D, q->H * C::D, C::D,
                        C::D, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TM_OK) return st;
  } else {
    mQ8 = mQ16;
  }
  ParamsC p;
  p.out = static_cast<__half*>(out->data);
  p.out_st = out->stride_t;
  p.out_sh = out->stride_h;
  p.q_scales = static_cast<const float*>(q->scales);
  p.k_tok_scale = static_cast<const __half*>(k->scales);
  p.v_tok_scale = static_cast<const __half*>(v->scales);
  p.bitmask = bitmask;
  p.mask_hs = mask_hs;
  p.cu = cu;
  p.cu_k = cu ? (cu_k ? cu_k : cu) : nullptr;
  p.Lq = q->T;
  p.Lk = k->T;
  p.Hq = static_cast<int>(q->H);
  p.Hkv = static_cast<int>(k->H);
  p.tile_m = tile_m;
  p.g = g;
  p.causal = causal ? 1 : 0;
  p.batch = cu ? batch : 1;
  const int64_t maxq = cu ? max_q : q->T;
  const int64_t maxk = cu ? max_k : k->T;
  p.max_lk = maxk;
  p.n_qt_max = static_cast<int>((maxq + tile_m - 1) / tile_m);
  p.W = tm_mask_words(maxk, 128, g);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(C::D)));
  p.err = DevErr{device_error_word()};
  const int64_t grid = static_cast<int64_t>(p.n_qt_max) * p.batch * p.Hq;
  if (grid == 0) return TM_OK;
  if (grid > 0x7fffffffLL) return TM_ERR_UNSUPPORTED;
  attn_cache_kernel<<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mQ16, mQ8, mKc, mVc, p);
  return check_cuda(cudaGetLastError());
}

}  // namespace tmk
