// tm_attn.cu -- fused tile-routed FP16/INT8 attention forward (tm_attn_fwd).
//
// TileMix (Lattice paper page), abstract: score tiles, one routing bit per
// (query tile, group of g key tiles), FP16 or INT8 score computation per
// group, both routes updating one online-softmax state; all legal groups are
// computed; GQA, variable-length batches and INT8 K/V caches.  The all-FP16
// case is fused SDPA as benchmarked in the MLX PR "Nax Refactor" tables.
//
// Kernel design (sm_100a, one CTA per (query tile, sequence, head)):
//   warp 4      TMA producer: Q (fp16, and int8 codes when the row has INT8
//               groups) once; per key tile either the fp16 K tile or the int8
//               K-code tile, chosen by the routing bit, plus the fp16 V tile,
//               into 2-stage rings of 128B-swizzled shared memory.
//   warp 5      tcgen05 issuer (one thread): S_j = Q K_j^T with kind::f16
//               (fp32 accumulate) or kind::i8 (s32 accumulate) into TMEM
//               (double-buffered S), then O += P_{j-1} V_{j-1} with P read
//               from TMEM (kind::f16, fp32 accumulate in TMEM).
//   warps 0-3   softmax, one query row per thread (TMEM lane = row): S row
//               from TMEM, int32 -> fp32 and dequantisation by
//               s_q * s_k * sigma for INT8 tiles, causal / ragged masking,
//               online max / sum with a lazy rescale of O (only when the row
//               max grows by more than 2^15), P rounded to fp16 and written back
//               over S in TMEM, and the final O / l epilogue.
// Every mbarrier wait is bounded (tm_device.cuh).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

// Which 128 x 128-tile launches with fp16 K / V take the kernel with one
// query tile per CTA and three score buffers (tm_attn3.cu) instead of the
// two-tile kernel (tm_attn2.cu): 0 none, 1 by use_one_tile_kernel_fp16
// below, 2 all.
#ifndef TM_SPLIT_KERNEL
#define TM_SPLIT_KERNEL 1
#endif
#include <atomic>

#include "tm_attn_internal.h"

namespace tmk {
namespace {

int device_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) ==
                                                   cudaSuccess && v > 0)
      sms = v;
    else
      return 148;
  }
  return sms;
}

// The choice between a two-query-tile kernel and its one-query-tile
// counterpart for the INT8-cache and FP8 launches and for all-FP16 rows of
// 64 or more key tiles (the fp16 path below takes the one-tile kernel's
// ping-pong form everywhere else).  Measured on B200 (a table of all-FP16
// MLX-shaped launches and the routing sweep): per tile the two-tile kernels
// are as fast as those one-tile ones on FP16 tiles and faster once INT8
// tiles are routed, but they have half as many CTAs.  The one-tile kernel is
// taken when the two-tile kernel would leave SMs idle (fewer CTAs than SMs),
// and for all-FP16 launches without a causal mask when its CTAs fill their
// last wave clearly better (causal launches already balance their waves by
// running the longest query tiles first).  sms: the GPU's SM count (0: the
// current device's).
std::atomic<int> g_attn_kernel{0};   // tm_set_attn_kernel

bool use_one_tile_kernel(int64_t n_qt, int64_t batch, int64_t hq, bool routed, bool causal, int64_t d = 128,
                         int64_t sms = 0) {
  const int choice = g_attn_kernel.load(std::memory_order_relaxed);
  if (choice != 0) return choice == 2;
  // At d = 64 a tile's MMAs are half as long while its softmax costs the
  // same, so the two-tile kernel's chain (softmax, P.V, next QK^T) leaves
  // the softmax waiting; the one-tile kernel's three score buffers and its
  // two independent softmax streams keep it busy.  Measured on the 24
  // MLX-shaped d = 64 runs: equal on one (1024^2, 32 heads, non-causal),
  // faster on the rest (up to 2.2x).
  if (d == 64) return true;
  if (sms <= 0) sms = device_sms();
  const int64_t pair_ctas = (n_qt + 1) / 2 * batch * hq, one_ctas = n_qt * batch * hq;
  // Fewer two-tile CTAs than SMs: the one-tile kernel, except for all-FP16
  // non-causal launches where the two-tile kernel still fills >= 80 % of the
  // SMs in one wave and the one-tile kernel would need a second (1024^2,
  // 32 heads: 0.032 against 0.035 ms; 2048^2, 16 heads: even).
  if (pair_ctas < sms)
    return routed || causal || 5 * pair_ctas < 4 * sms || one_ctas <= sms;
  if (routed || causal) return false;
  auto fill = [&](int64_t ctas) { return static_cast<double>(ctas) / (((ctas + sms - 1) / sms) * sms); };
  return fill(one_ctas) > 1.1 * fill(pair_ctas);
}

// The choice for fp16 K / V without the FP8 route, where the one-tile
// kernel runs its ping-pong softmax at d = 128 (tm_attn3.cu): measured on
// B200 it beats the two-tile kernel on routed launches (routing sweep,
// L = 16384: 2.03 / 2.05 / 2.01 ms against 2.13 / 2.21 / 2.08 ms at INT8
// group probability 0 / 0.75 / 1) and on all-FP16 rows of fewer than 64 key
// tiles (4096^2 32 heads non-causal 0.261 against 0.305 ms, causal 0.159
// against 0.163; 2048^2 and 1024^2 equal or faster).  All-FP16 rows of 64 or
// more key tiles keep the rule above: there the two-tile kernel's chunked
// mode is faster (routing-sweep shape without a mask: 2.08 against 2.21 ms).
bool use_one_tile_kernel_fp16(int64_t n_qt, int64_t n_kt, int64_t batch, int64_t hq, bool routed, bool causal,
                              int64_t d, int64_t sms = 0) {
  const int choice = g_attn_kernel.load(std::memory_order_relaxed);
  if (choice != 0) return choice == 2;
  if (d == 128 && (routed || n_kt < 64)) return true;
  return use_one_tile_kernel(n_qt, batch, hq, routed, causal, d, sms);
}

}  // namespace
}  // namespace tmk

extern "C" tm_status tm_set_attn_kernel(int32_t choice) {
  if (choice < 0 || choice > 2) return TM_ERR_INVALID_ARG;
  tmk::g_attn_kernel.store(choice, std::memory_order_relaxed);
  return TM_OK;
}

extern "C" int32_t tm_attn_kernel_choice(int64_t max_q, int64_t max_k, int32_t batch, int32_t hq, int32_t d,
                                         int32_t routed, int32_t causal, int32_t sm_count) {
  if (max_q <= 0 || max_k <= 0 || batch <= 0 || hq <= 0 || (d != 64 && d != 128) || sm_count < 0) return 0;
  const int64_t n_qt = (max_q + 127) / 128, n_kt = (max_k + 127) / 128;
  return tmk::use_one_tile_kernel_fp16(n_qt, n_kt, batch, hq, routed != 0, causal != 0, d, sm_count) ? 2 : 1;
}
#include "tm_device.cuh"
#include "tm_host.h"

namespace tmk {
namespace {

template <int D, int BN>
struct Cfg {
  static constexpr int BM = 128;                 // MMA rows (query tile of 128, or 64 + unused)
  static constexpr int NK = 2, NV = 2;           // ring depths
  static constexpr int Q16_HALF = BM * 128;      // bytes of one 64-column fp16 slab of Q
  static constexpr int KV16_HALF = BN * 128;     // bytes of one 64-column fp16 slab of K / V
  static constexpr int Q16_BYTES = BM * D * 2;
  static constexpr int Q8_BYTES = BM * D;
  static constexpr int K_STAGE = BN * D * 2;
  static constexpr int V_STAGE = BN * D * 2;
  static constexpr int OFF_Q16 = 0;
  static constexpr int OFF_Q8 = OFF_Q16 + Q16_BYTES;
  static constexpr int OFF_K = OFF_Q8 + Q8_BYTES;
  static constexpr int OFF_V = OFF_K + NK * K_STAGE;
  static constexpr int OFF_BAR = OFF_V + NV * V_STAGE;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;   // + alignment slack
  static constexpr uint32_t TMEM_COLS = (2 * BN + D <= 256) ? 256u : 512u;
  static constexpr uint32_t O_COL = 2 * BN;
  static constexpr uint32_t IDESC_S16 = idesc_f16(BM, BN, false);
  static constexpr uint32_t IDESC_S8 = idesc_i8(BM, BN);
  static constexpr uint32_t IDESC_PV = idesc_f16(BM, D, true);
  static constexpr uint32_t Q8_SWZ = (D == 128) ? kSwizzle128 : kSwizzle64;
  static constexpr uint32_t Q8_SBO = (D == 128) ? 1024u : 512u;
};

// Barrier slots (uint64 each) inside the barrier block.
enum {
  B_QFULL = 0,
  B_KFULL = 1,   // +NK
  B_KEMPTY = 3,  // +NK
  B_VFULL = 5,   // +NV
  B_VEMPTY = 7,  // +NV
  B_SFULL = 9,   // +2
  B_PFULL = 11,  // +2
  B_ODONE = 13,
  B_DRAIN = 14,
  B_COUNT = 15
};

struct Params {
  __half* out;
  int64_t out_st, out_sh;
  const float* q_scales;   // [n_qtiles, Hq]
  const float* k_scales;   // [n_ktiles, Hkv]
  const uint32_t* bitmask;
  int64_t mask_hs;
  int W;
  const int32_t* cu;
  const int32_t* cu_k;     // key offsets (= cu unless separate)
  int64_t max_lk;          // longest key row the launch was sized for
  int64_t Lq, Lk;          // lengths without cu_seqlens
  int Hq, Hkv, tile_m, g, causal, n_qt_max, batch;
  float scale_log2;        // sigma * log2(e)
  DevErr err;
};

__device__ __forceinline__ bool route_int8(const uint32_t* row, int g, int j) {
  if (row == nullptr) return false;
  const int G = j / g;
  return (__ldg(row + (G >> 5)) >> (G & 31)) & 1u;
}

template <int D, int BN>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ16, const __grid_constant__ CUtensorMap tmQ8,
                    const __grid_constant__ CUtensorMap tmK16, const __grid_constant__ CUtensorMap tmK8,
                    const __grid_constant__ CUtensorMap tmV16, const Params p) {
  using C = Cfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;
  const uint32_t sQ16 = sbase + C::OFF_Q16;
  const uint32_t sQ8 = sbase + C::OFF_Q8;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * B_COUNT + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: heaviest query tiles first (causal), heads fastest
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
  if (p.cu != nullptr && I == 0 && threadIdx.x == 0 &&
      Lq > static_cast<int64_t>(p.n_qt_max) * p.tile_m)
    dev_error(p.err, TM_DEVERR_SEQLEN);
  if (static_cast<int64_t>(I) * p.tile_m >= Lq) return;   // whole CTA: no setup done yet

  const int rows_valid = static_cast<int>(min(static_cast<int64_t>(p.tile_m), Lq - static_cast<int64_t>(I) * p.tile_m));
  const int64_t i_last = static_cast<int64_t>(I) * p.tile_m + rows_valid - 1;
  int64_t jmax = Lk - 1;
  if (p.causal) jmax = min(jmax, i_last + Lk - Lq);
  const int nJ = (Lk <= 0 || jmax < 0) ? 0 : static_cast<int>(jmax / BN + 1);
  const int64_t ig = sq.tile_base + I;
  const int hk = h / (p.Hq / p.Hkv);
  const uint32_t* mrow = p.bitmask ? p.bitmask + static_cast<int64_t>(h) * p.mask_hs + ig * p.W : nullptr;
  const int64_t qrow0 = sq.start + static_cast<int64_t>(I) * p.tile_m;

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < C::NK; ++s) { mbar_init(bar(B_KFULL + s), 1); mbar_init(bar(B_KEMPTY + s), 1); }
    for (int s = 0; s < C::NV; ++s) { mbar_init(bar(B_VFULL + s), 1); mbar_init(bar(B_VEMPTY + s), 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(bar(B_SFULL + s), 1); mbar_init(bar(B_PFULL + s), 128); }
    mbar_init(bar(B_ODONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmQ16);
    prefetch_tmap(&tmK16);
    prefetch_tmap(&tmV16);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ======================= TMA producer =======================
    if (lane == 0 && nJ > 0) {
      bool any8 = false;
      if (mrow != nullptr)
        for (int w = 0; w < p.W; ++w) any8 |= (__ldg(mrow + w) != 0u);
      mbar_arrive_expect_tx(bar(B_QFULL), C::Q16_BYTES + (any8 ? C::Q8_BYTES : 0));
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh)
        tma_load_3d(sQ16 + hh * C::Q16_HALF, &tmQ16, bar(B_QFULL), hh * 64, h, static_cast<int32_t>(qrow0));
      if (any8) tma_load_3d(sQ8, &tmQ8, bar(B_QFULL), 0, h, static_cast<int32_t>(qrow0));
      int nk_issued = 0, nv_issued = 0;
      for (int j = 0; j < nJ; ++j) {
        const bool i8 = route_int8(mrow, p.g, j);
        const int32_t krow = static_cast<int32_t>(kstart + static_cast<int64_t>(j) * BN);
        const int ks = j % C::NK, kn = j / C::NK;
        if (kn > 0 && !mbar_wait(bar(B_KEMPTY + ks), (kn - 1) & 1, p.err, abort_flag)) break;
        const uint32_t kdst = sK + ks * C::K_STAGE;
        if (i8) {
          mbar_arrive_expect_tx(bar(B_KFULL + ks), BN * D);
          tma_load_3d(kdst, &tmK8, bar(B_KFULL + ks), 0, hk, krow);
        } else {
          mbar_arrive_expect_tx(bar(B_KFULL + ks), BN * D * 2);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(kdst + hh * C::KV16_HALF, &tmK16, bar(B_KFULL + ks), hh * 64, hk, krow);
        }
        ++nk_issued;
        const int vs = j % C::NV, vn = j / C::NV;
        if (vn > 0 && !mbar_wait(bar(B_VEMPTY + vs), (vn - 1) & 1, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(bar(B_VFULL + vs), BN * D * 2);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(sV + vs * C::V_STAGE + hh * C::KV16_HALF, &tmV16, bar(B_VFULL + vs), hh * 64, hk, krow);
        ++nv_issued;
      }
      // Drain: every issued copy has landed before the CTA may exit.
      volatile int never = 0;
      mbar_wait(bar(B_QFULL), 0, p.err, &never);
      for (int s = 0; s < C::NK; ++s) {
        const int cnt = nk_issued > s ? (nk_issued - 1 - s) / C::NK + 1 : 0;
        if (cnt > 0) mbar_wait(bar(B_KFULL + s), (cnt - 1) & 1, p.err, &never);
      }
      for (int s = 0; s < C::NV; ++s) {
        const int cnt = nv_issued > s ? (nv_issued - 1 - s) / C::NV + 1 : 0;
        if (cnt > 0) mbar_wait(bar(B_VFULL + s), (cnt - 1) & 1, p.err, &never);
      }
    }
  } else if (warp == 5) {
    // ======================= tcgen05 issuer =======================
    if (lane == 0 && nJ > 0) {
      bool ok = mbar_wait(bar(B_QFULL), 0, p.err, abort_flag);
      tc_fence_after();
      auto issue_pv = [&](int t) -> bool {
        if (!mbar_wait(bar(B_PFULL + (t & 1)), (t >> 1) & 1, p.err, abort_flag)) return false;
        const int vs = t % C::NV;
        if (!mbar_wait(bar(B_VFULL + vs), (t / C::NV) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t a_tmem = tmem + static_cast<uint32_t>(t & 1) * BN;
        const uint32_t vbase = sV + vs * C::V_STAGE;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = smem_desc(vbase + kk * 2048, C::KV16_HALF, 1024, kSwizzle128);
          mma_f16_ts(tmem + C::O_COL, a_tmem + kk * 8, bdesc, C::IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_ODONE));
        tc_commit(bar(B_VEMPTY + vs));
        return true;
      };
      for (int j = 0; ok && j < nJ; ++j) {
        const bool i8 = route_int8(mrow, p.g, j);
        const int ks = j % C::NK;
        if (!mbar_wait(bar(B_KFULL + ks), (j / C::NK) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(j & 1) * BN;
        const uint32_t kbase = sK + ks * C::K_STAGE;
        if (i8) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t ad = smem_desc(sQ8 + kk * 32, 16, C::Q8_SBO, C::Q8_SWZ);
            const uint64_t bd = smem_desc(kbase + kk * 32, 16, C::Q8_SBO, C::Q8_SWZ);
            mma_i8_ss(d_tmem, ad, bd, C::IDESC_S8, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 0u + (kk & 3) * 32;
            const uint64_t ad = smem_desc(sQ16 + (kk >> 2) * C::Q16_HALF + off, 16, 1024, kSwizzle128);
            const uint64_t bd = smem_desc(kbase + (kk >> 2) * C::KV16_HALF + off, 16, 1024, kSwizzle128);
            mma_f16_ss(d_tmem, ad, bd, C::IDESC_S16, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit(bar(B_SFULL + (j & 1)));
        tc_commit(bar(B_KEMPTY + ks));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(nJ - 1);
      // Drain: all issued tcgen05 work completes before TMEM is released.
      tc_commit(bar(B_DRAIN));
      volatile int never = 0;
      mbar_wait(bar(B_DRAIN), 0, p.err, &never);
    }
  } else {
    // ======================= softmax (warps 0-3) =======================
    const int r = threadIdx.x;                       // query row in the tile = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool row_ok = r < rows_valid;
    const int64_t i_row = static_cast<int64_t>(I) * p.tile_m + r;
    int64_t lim = -1;                                // last visible key of this row
    if (row_ok) lim = p.causal ? min(Lk - 1, i_row + Lk - Lq) : Lk - 1;
    float c8_row = 0.f;
    if (mrow != nullptr) c8_row = __ldg(p.q_scales + ig * p.Hq + h) * p.scale_log2;
    const SeqInfo sk = seq_info(p.cu_k, b, p.Lk, BN);  // key-tile numbering of this sequence
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nJ; ++j) {
      const bool i8 = route_int8(mrow, p.g, j);
      float c = p.scale_log2;
      // INT8 tile: S = acc * s_q * s_k * sigma; kept > 0 so that masked -inf
      // scores stay -inf (an all-zero tile has acc = 0 and gives S = 0).
      if (i8) c = fmaxf(c8_row * __ldg(p.k_scales + (sk.tile_base + j) * p.Hkv + hk), 1e-30f);
      if (!mbar_wait(bar(B_SFULL + (j & 1)), (j >> 1) & 1, p.err, abort_flag)) { ok = false; break; }
      tc_fence_after();
      __syncwarp();
      float x[BN];
      {
        uint32_t u[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc)
          tmem_ld32p(lane_addr + static_cast<uint32_t>(j & 1) * BN + cc * 32, u + cc * 32);
        tmem_wait_ld_regs<BN>(u);
        if (i8) {
          // exact int32 -> fp32 for |acc| < 2^22: add the bits of 1.5 * 2^23
#pragma unroll
          for (int e = 0; e < BN; ++e) x[e] = __int_as_float(static_cast<int>(u[e]) + 0x4B400000) - 12582912.0f;
        } else {
#pragma unroll
          for (int e = 0; e < BN; ++e) x[e] = __uint_as_float(u[e]);
        }
      }
      const int64_t nv64 = lim - static_cast<int64_t>(j) * BN + 1;
      const int nv = nv64 <= 0 ? 0 : (nv64 >= BN ? BN : static_cast<int>(nv64));
      if (!__all_sync(0xffffffffu, nv == BN)) {
#pragma unroll
        for (int e = 0; e < BN; ++e) x[e] = (e < nv) ? x[e] : -INFINITY;
      }
      float alpha = 1.f;
      if (nv > 0) {
        const float mt = row_max<BN>(x) * c;
        if (mt > m_used + kLazyRescaleLog2) {   // lazy rescale
          alpha = ex2_approx(m_used - mt);
          m_used = mt;
        }
      }
      const float msub = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t pk[BN / 2];
      float acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll
      for (int e = 0; e < BN; e += 2) {
        const float p0 = ex2_approx(fmaf(x[e], c, -msub));
        const float p1 = ex2_approx(fmaf(x[e + 1], c, -msub));
        acc[(e >> 1) & 7] += p0 + p1;
        pk[e >> 1] = pack_half2(p0, p1);
      }
      l = l * alpha + ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      if (j > 0) {
        // O holds sum_{t<j} P_t V_t once PV_{j-1} has completed.
        if (!mbar_wait(bar(B_ODONE), (j - 1) & 1, p.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        __syncwarp();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          uint32_t o[D];
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_ld32p(lane_addr + C::O_COL + cc * 32, o + cc * 32);
          tmem_wait_ld_regs<D>(o);
#pragma unroll
          for (int e = 0; e < D; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_st32p(lane_addr + C::O_COL + cc * 32, o + cc * 32);
        }
      }
      __syncwarp();
#pragma unroll
      for (int cc = 0; cc < BN / 64; ++cc)
        tmem_st32p(lane_addr + static_cast<uint32_t>(j & 1) * BN + cc * 32, pk + cc * 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + (j & 1)));
    }
    // ---- epilogue: out = O / l (0 for rows without a visible key)
    bool have_o = false;
    if (ok && nJ > 0) {
      have_o = mbar_wait(bar(B_ODONE), (nJ - 1) & 1, p.err, abort_flag);
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
        reinterpret_cast<uint4*>(orow)[cc] = pkt;
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

std::mutex g_attr_mu;

template <int D, int BN>
tm_status launch(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                 const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                 const uint32_t* bitmask,
                 int64_t mask_hs, int32_t tile_m, int32_t g, int32_t causal, cudaStream_t stream) {
  using C = Cfg<D, BN>;
  static bool attr_done = false;
  {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (!attr_done) {
      tm_status st = check_cuda(cudaFuncSetAttribute(attn_fwd_kernel<D, BN>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     C::SMEM_BYTES));
      if (st != TM_OK) return st;
      attr_done = true;
    }
  }
  CUtensorMap mQ16, mQ8, mK16, mK8, mV16;
  tm_status st;
  st = encode_thd_map(&mQ16, q->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, q->T, q->H, D, q->stride_t,
                      q->stride_h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mK16, k->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, k->T, k->H, D, k->stride_t,
                      k->stride_h, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mV16, v->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, v->T, v->H, D, v->stride_t,
                      v->stride_h, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  const CUtensorMapSwizzle swz8 = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (bitmask != nullptr) {
    st = encode_thd_map(&mQ8, q->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->T, q->H, D, q->H * D, D,
                        D, 128, swz8);
    if (st != TM_OK) return st;
    st = encode_thd_map(&mK8, k->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k->T, k->H, D, k->H * D, D,
                        D, BN, swz8);
    if (st != TM_OK) return st;
  } else {
    mQ8 = mQ16;
    mK8 = mK16;
  }
  Params p;
  p.out = static_cast<__half*>(out->data);
  p.out_st = out->stride_t;
  p.out_sh = out->stride_h;
  p.q_scales = static_cast<const float*>(q->scales);
  p.k_scales = static_cast<const float*>(k->scales);
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
  p.W = tm_mask_words(maxk, BN, g);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(D)));
  p.err = DevErr{device_error_word()};
  const int64_t grid = static_cast<int64_t>(p.n_qt_max) * p.batch * p.Hq;
  if (grid == 0) return TM_OK;
  if (grid > 0x7fffffffLL) return TM_ERR_UNSUPPORTED;
  attn_fwd_kernel<D, BN><<<static_cast<unsigned>(grid), 192, C::SMEM_BYTES, stream>>>(mQ16, mQ8, mK16,
                                                                                      mK8, mV16, p);
  return check_cuda(cudaGetLastError());
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tm_status check_fp16(const tm_tensor* t, int64_t d) {
  if (t == nullptr || t->data == nullptr || !aligned16(t->data)) return TM_ERR_INVALID_ARG;
  if (t->T < 0 || t->H <= 0 || t->d != d) return TM_ERR_INVALID_ARG;
  if (t->stride_h < d || (t->stride_h % 8) || (t->stride_t % 8)) return TM_ERR_INVALID_ARG;
  if (t->H > 1 && t->stride_t < t->stride_h * (t->H - 1) + d) return TM_ERR_INVALID_ARG;
  if (t->H == 1 && t->stride_t < d) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

}  // namespace
}  // namespace tmk

namespace tmk {
namespace {

// Shared body of tm_attn_fwd (cu_k null: keys use the query offsets) and
// tm_attn_fwd_varlen (separate key offsets).
tm_status attn_fwd_impl(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                        const int32_t* cu_seqlens, const int32_t* cu_k, int32_t batch, int32_t max_seqlen,
                        int32_t max_k, const uint32_t* bitmask, int64_t mask_head_stride, int32_t tile_m,
                        int32_t tile_n, int32_t g, int32_t causal, void* stream, const Fp8Route* f8 = nullptr,
                        void* cache_ws = nullptr, int64_t cache_ws_bytes = 0) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return TM_ERR_INVALID_ARG;
  const int64_t D = q->d;
  if (D != 64 && D != 128) return TM_ERR_UNSUPPORTED;
  if ((tile_m != 64 && tile_m != 128) || (tile_n != 64 && tile_n != 128)) return TM_ERR_UNSUPPORTED;
  if (g < 1 || mask_head_stride < 0) return TM_ERR_INVALID_ARG;
  tm_status st = check_fp16(q, D);
  if (st != TM_OK) return st;
  st = check_fp16(out, D);
  if (st != TM_OK) return st;
  if (out->T != q->T || out->H != q->H) return TM_ERR_INVALID_ARG;
  if (q->H % k->H != 0 || q->H > 65535 || k->H <= 0) return TM_ERR_INVALID_ARG;
  if (cu_seqlens != nullptr && (batch <= 0 || max_seqlen <= 0)) return TM_ERR_INVALID_ARG;
  if (cu_k != nullptr && (cu_seqlens == nullptr || max_k <= 0)) return TM_ERR_INVALID_ARG;
  // with shared offsets the key rows are the query rows
  const bool shared = cu_seqlens != nullptr && cu_k == nullptr;
  if (shared) max_k = max_seqlen;
  if (bitmask != nullptr) {
    if (reinterpret_cast<uintptr_t>(bitmask) & 3u) return TM_ERR_INVALID_ARG;
    if (q->codes == nullptr || !aligned16(q->codes) || q->scale_kind != TM_SCALE_TILE || q->scales == nullptr)
      return TM_ERR_INVALID_ARG;
  }
  const bool cache = (k->scale_kind == TM_SCALE_TOKEN) || (v->scale_kind == TM_SCALE_TOKEN);
  if (f8 != nullptr) {
    // the FP8 route: d = 128, 128 x 128 tiles, fp16 K / V, one-tile kernel
    if (cache || D != 128 || tile_m != 128 || tile_n != 128) return TM_ERR_UNSUPPORTED;
    if (f8->bitmask == nullptr || (reinterpret_cast<uintptr_t>(f8->bitmask) & 3u)) return TM_ERR_INVALID_ARG;
    if (f8->q_codes == nullptr || f8->k_codes == nullptr || !aligned16(f8->q_codes) || !aligned16(f8->k_codes))
      return TM_ERR_INVALID_ARG;
    if (f8->q_scales == nullptr || f8->k_scales == nullptr || (reinterpret_cast<uintptr_t>(f8->q_scales) & 3u) ||
        (reinterpret_cast<uintptr_t>(f8->k_scales) & 3u))
      return TM_ERR_INVALID_ARG;
  }
  if (cache) {
    // INT8 K/V cache: both K and V as codes + per-(token, head) fp16 scales.
    if (k->scale_kind != TM_SCALE_TOKEN || v->scale_kind != TM_SCALE_TOKEN) return TM_ERR_INVALID_ARG;
    if (k->codes == nullptr || v->codes == nullptr || k->scales == nullptr || v->scales == nullptr)
      return TM_ERR_INVALID_ARG;
    if (!aligned16(k->codes) || !aligned16(v->codes) || (reinterpret_cast<uintptr_t>(k->scales) & 1u) ||
        (reinterpret_cast<uintptr_t>(v->scales) & 1u))
      return TM_ERR_INVALID_ARG;
    if (k->T != v->T || k->H != v->H || k->d != D || v->d != D || k->T < 0) return TM_ERR_INVALID_ARG;
    if (shared && k->T != q->T) return TM_ERR_INVALID_ARG;
    if (D != 128 || tile_n != 128) return TM_ERR_UNSUPPORTED;
    if (cache_ws != nullptr && tile_m == 128) {
      // The cache expanded once into the caller's workspace (its fp16 view
      // and per-token K scales by key tile), then attention over the fp16
      // view: all-FP16 launches as for fp16 K / V, routed launches on the
      // two-query-tile kernel with the INT8 route's scales per key token.
      const CacheWsLayout L = cache_ws_layout(k->T, static_cast<int32_t>(k->H), cu_seqlens ? batch : 0);
      if (cache_ws_bytes < L.bytes || (reinterpret_cast<uintptr_t>(cache_ws) & 255u)) return TM_ERR_INVALID_ARG;
      const int32_t* key_cu = cu_seqlens ? (cu_k ? cu_k : cu_seqlens) : nullptr;
      cudaStream_t s = as_stream(stream);
      st = launch_cache_expand(k, v, key_cu, batch, max_k, cache_ws, L, s);
      if (st != TM_OK) return st;
      uint8_t* ws = static_cast<uint8_t*>(cache_ws);
      tm_tensor kk = *k, vv = *v;
      kk.data = ws + L.off_k16;
      vv.data = ws + L.off_v16;
      kk.stride_t = vv.stride_t = k->H * 128;
      kk.stride_h = vv.stride_h = 128;
      kk.scales = vv.scales = nullptr;
      kk.scale_kind = vv.scale_kind = TM_SCALE_NONE;
      vv.codes = nullptr;
      if (bitmask == nullptr) {
        kk.codes = nullptr;
        return attn_fwd_impl(q, &kk, &vv, out, cu_seqlens, cu_k, batch, max_seqlen, cu_k ? max_k : 0, nullptr,
                             mask_head_stride, tile_m, tile_n, g, causal, stream);
      }
      return launch_attn_pair_toks(q, &kk, &vv, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask,
                                   mask_head_stride, g, causal, reinterpret_cast<const float*>(ws + L.off_kst),
                                   L.kst_tiles, s);
    }
    // 128-row query tiles: two per CTA, unless that leaves SMs idle or the
    // one-tile kernel is chosen (tm_set_attn_kernel)
    const int64_t n_qt = ((cu_seqlens ? max_seqlen : q->T) + 127) / 128;
    if (tile_m == 128 && !use_one_tile_kernel(n_qt, cu_seqlens ? batch : 1, q->H, true, causal != 0))
      return launch_attn_pair_cache(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask,
                                    mask_head_stride, g, causal, as_stream(stream));
    return launch_attn_cache(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                             tile_m, g, causal, as_stream(stream));
  }
  st = check_fp16(k, D);
  if (st != TM_OK) return st;
  st = check_fp16(v, D);
  if (st != TM_OK) return st;
  if (k->T != v->T || k->H != v->H) return TM_ERR_INVALID_ARG;
  if (q->H % k->H != 0 || q->H > 65535) return TM_ERR_INVALID_ARG;
  if (shared && k->T != q->T) return TM_ERR_INVALID_ARG;
  if (bitmask != nullptr) {
    if (k->codes == nullptr || !aligned16(k->codes) || k->scale_kind != TM_SCALE_TILE || k->scales == nullptr)
      return TM_ERR_INVALID_ARG;
  }
  cudaStream_t s = as_stream(stream);
  if (f8 != nullptr) {
    // FP8 and FP16 only (no INT8 plane): the two-query-tile kernel with its
    // 8-bit route in E4M3, unless that leaves SMs idle or the one-tile
    // kernel is chosen; three-way routing runs on the one-tile kernel
    const int64_t n_qt = ((cu_seqlens ? max_seqlen : q->T) + 127) / 128;
    if (bitmask == nullptr && !use_one_tile_kernel(n_qt, cu_seqlens ? batch : 1, q->H, true, causal != 0)) {
      tm_tensor qq = *q, kk = *k;
      qq.codes = reinterpret_cast<const int8_t*>(f8->q_codes);
      qq.scales = f8->q_scales;
      qq.scale_kind = TM_SCALE_TILE;
      kk.codes = reinterpret_cast<const int8_t*>(f8->k_codes);
      kk.scales = f8->k_scales;
      kk.scale_kind = TM_SCALE_TILE;
      return launch_attn_pair_fp8(&qq, &kk, v, out, cu_seqlens, batch, max_seqlen, f8->bitmask, mask_head_stride,
                                  g, causal, s);
    }
    return launch_attn_split(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride, g,
                             causal, s, f8);
  }
  if (tile_m == 128 && tile_n == 128) {
    const int64_t n_qt = ((cu_seqlens ? max_seqlen : q->T) + 127) / 128;
    const int64_t n_kt = ((cu_seqlens ? max_k : k->T) + 127) / 128;
    if (TM_SPLIT_KERNEL == 2 ||
        (TM_SPLIT_KERNEL == 1 && use_one_tile_kernel_fp16(n_qt, n_kt, cu_seqlens ? batch : 1, q->H,
                                                          bitmask != nullptr, causal != 0, D)))
      return launch_attn_split(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                               g, causal, s);
    return launch_attn_pair(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                            g, causal, s);
  }
  if (D == 128) {
    if (tile_n == 128)
      return launch<128, 128>(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                              tile_m, g, causal, s);
    return launch<128, 64>(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                           tile_m, g, causal, s);
  }
  if (tile_n == 128)
    return launch<64, 128>(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                           tile_m, g, causal, s);
  return launch<64, 64>(q, k, v, out, cu_seqlens, cu_k, batch, max_seqlen, max_k, bitmask, mask_head_stride,
                        tile_m, g, causal, s);
}

}  // namespace
}  // namespace tmk

extern "C" tm_status tm_attn_fwd(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v,
                                 tm_tensor* out, const int32_t* cu_seqlens, int32_t batch,
                                 int32_t max_seqlen, const uint32_t* bitmask,
                                 int64_t mask_head_stride, int32_t tile_m, int32_t tile_n,
                                 int32_t g, int32_t causal, void* stream) {
  return tmk::attn_fwd_impl(q, k, v, out, cu_seqlens, nullptr, batch, max_seqlen, 0, bitmask, mask_head_stride,
                            tile_m, tile_n, g, causal, stream);
}

extern "C" tm_status tm_attn_fwd_varlen(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v,
                                        tm_tensor* out, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int32_t batch, int32_t max_seqlen_q,
                                        int32_t max_seqlen_k, const uint32_t* bitmask,
                                        int64_t mask_head_stride, int32_t tile_m, int32_t tile_n, int32_t g,
                                        int32_t causal, void* stream) {
  if (cu_seqlens_q == nullptr || cu_seqlens_k == nullptr) return TM_ERR_INVALID_ARG;
  return tmk::attn_fwd_impl(q, k, v, out, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q, max_seqlen_k, bitmask,
                            mask_head_stride, tile_m, tile_n, g, causal, stream);
}

extern "C" tm_status tm_attn_fwd_cache_ws(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v,
                                          tm_tensor* out, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                          int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                          const uint32_t* bitmask, int64_t mask_head_stride, int32_t tile_m,
                                          int32_t tile_n, int32_t g, int32_t causal, void* workspace,
                                          int64_t workspace_bytes, void* stream) {
  if (k == nullptr || v == nullptr || k->scale_kind != TM_SCALE_TOKEN || v->scale_kind != TM_SCALE_TOKEN)
    return TM_ERR_INVALID_ARG;
  if (workspace == nullptr) return TM_ERR_INVALID_ARG;
  if (cu_seqlens_k != nullptr && cu_seqlens_q == nullptr) return TM_ERR_INVALID_ARG;
  return tmk::attn_fwd_impl(q, k, v, out, cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q,
                            cu_seqlens_k ? max_seqlen_k : 0, bitmask, mask_head_stride, tile_m, tile_n, g, causal,
                            stream, nullptr, workspace, workspace_bytes);
}

extern "C" tm_status tm_attn_fwd_fp8(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                                     const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen,
                                     const uint32_t* bitmask, const uint32_t* bitmask_fp8, int64_t mask_head_stride,
                                     const uint8_t* q_fp8_codes, const float* q_fp8_scales,
                                     const uint8_t* k_fp8_codes, const float* k_fp8_scales, int32_t g,
                                     int32_t causal, void* stream) {
  const tmk::Fp8Route f8{bitmask_fp8, q_fp8_codes, q_fp8_scales, k_fp8_codes, k_fp8_scales};
  return tmk::attn_fwd_impl(q, k, v, out, cu_seqlens, nullptr, batch, max_seqlen, 0, bitmask, mask_head_stride, 128,
                            128, g, causal, stream, &f8);
}
