// tm_attn3.cu -- fused tile-routed attention, one 128-row query tile per CTA
// with three score buffers in TMEM (d = 128 or 64, 128-key tiles).
//
// TileMix (Lattice paper page), abstract: score tiles routed per group of g
// key tiles to an FP16 or an INT8 QK^T, both feeding one online-softmax state.
//
// Why this layout.  Measured on B200, a group of tcgen05 MMAs started on an
// idle tensor pipe takes about 600 cycles longer than the same MMAs back to
// back (pipeline fill, drain, commit and wake-up).  When the score tile S and
// its probabilities P share TMEM columns, a query tile runs the chain
//     softmax(j) -> P.V(j) -> QK^T(j+1) -> softmax(j+1)
// and pays that latency once per key tile.  Here the 512 TMEM columns hold
// the fp32 accumulator O (128 columns; two of 64 at d = 64) and three score
// buffers, so the tensor pipe computes QK^T(j+1) and QK^T(j+2) ahead while
// the softmax works on S(j):
//
//   * S(j) goes to buffer j mod 3.  Two softmax warpgroups (one query row
//     per thread, warpgroup h = warps 4h .. 4h+3) take alternate score
//     tiles, those with j mod 2 == h, in one of two forms:
//   * at d = 128 (ping-pong) both accumulate into one O (128 columns).  The
//     running max m (raised lazily, kLazyRescaleLog2) is handed from tile to
//     tile in key order: after loading S(j) and its row maxima, tile j's
//     warpgroup waits until P(j-1) is stored, reads the m that tile j-1
//     published in shared memory, raises it if tile j needs it (rescaling O
//     once P.V(j-1) has completed) and publishes its own.  So the two
//     warpgroups' exponentials alternate while one's loads and maxima
//     overlap the other's exponentials, and every P.V adds into O against
//     the reference a single stream would hold.  Each warpgroup keeps its
//     row sum against the reference of its own last tile; the epilogue
//     brings both to the final one;
//   * at d = 64 (dual stream) each warpgroup keeps its own running max, row
//     sum and O (O of warpgroup h in TMEM columns [64h, 64h+64)) and never
//     waits for the other; the epilogue merges the two streams.  (At
//     d = 128 two O accumulators and three score buffers would need 640 of
//     the 512 TMEM columns.)
//   * with the FP8 route (three-way routing, d = 128) the keys of each score
//     tile are instead split between the warpgroups (warpgroup h owns keys
//     [64h, 64h+64)); they exchange the tile's row maxima through shared
//     memory, so both rescale against one running max, each sums its half
//     of the row sum and rescales its half of O's columns;
//   * each warpgroup overwrites the first half of its score columns with
//     its P as fp16 (ping-pong: 32 columns at a time, as they are computed);
//     once the tile's P is complete, P.V(j) is one group of eight MMAs into
//     O (dual stream: into the O of warpgroup j mod 2), and
//     QK^T(j+3) follows it into the same buffer (the tensor pipe runs them
//     in order);
//   * K and V reach shared memory through two rings of 32 KB slots (three K
//     slots holding the int8 or the fp16 K tile by route, two V slots), each
//     slot released by a tcgen05.commit once the MMAs reading it completed,
//     so K prefetch never waits for a P.V;
//   * the softmax arithmetic is the same as in the two-tile kernel (packed
//     fp32 pairs; 3 of every 8 exp2 pairs -- 2 at d = 64 -- as a degree-3
//     minimax polynomial on the FMA pipe, the rest on MUFU.ex2).
// Every mbarrier wait is bounded (tm_device.cuh).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tm_attn_internal.h"
#include "tm_device.cuh"
#include "tm_host.h"

#ifdef TM_TRACE
extern "C" int tm_debug_trace_read_split(unsigned long long* host, unsigned int block) {
  if (host == nullptr) {
    static unsigned long long zero[TM_TRACE_ROLES][TM_TRACE_EVENTS];
    if (cudaMemcpyToSymbol(g_tm_trace, zero, sizeof(zero)) != cudaSuccess) return -1;
    return cudaMemcpyToSymbol(g_tm_trace_block, &block, sizeof(block)) == cudaSuccess ? 0 : -1;
  }
  return cudaMemcpyFromSymbol(host, g_tm_trace, sizeof(g_tm_trace)) == cudaSuccess ? 0 : -1;
}
#endif

// Softmax phase profile (compiled only with TM_PHASES and TM_TRACE): the
// first thread of each warpgroup sums SM-clock deltas per phase.
#ifdef TM_PHASES
#define TM3_PH_DECL long long tm_ph[8] = {0, 0, 0, 0, 0, 0, 0, 0}; long long tm_ph_t = clock64();
#define TM3_PH(i) do { const long long tm_now = clock64(); tm_ph[i] += tm_now - tm_ph_t; tm_ph_t = tm_now; } while (0)
#else
#define TM3_PH_DECL
#define TM3_PH(i) do { } while (0)
#endif

namespace tmk {
namespace {

template <int D_, bool F8>
struct Cfg3 {
  // DS (dual stream, d = 64): warpgroup h takes the whole key tiles j with
  // j mod 2 == h, each warpgroup with its own running max, row sum and O
  // (two 64-column accumulators), merged in the epilogue.  At d = 128 two O
  // accumulators and three score buffers would need 640 TMEM columns.
  static constexpr bool DS = D_ == 64;
  // PP (ping-pong, d = 128 without the FP8 route): warpgroup h also takes
  // the whole key tiles with j mod 2 == h, but both accumulate into one O.
  // The running max is handed from tile to tile in key order: before its
  // exponentials, tile j's warpgroup waits until tile j-1's P is stored and
  // takes that tile's reference max (raising it lazily, as one stream
  // would), so every P.V adds into O against one reference.
  static constexpr bool PP = D_ == 128 && !F8;
  static constexpr bool ALT = DS || PP;                         // warpgroups take alternate key tiles
  static constexpr int D = D_, BM = 128, BN = 128;
  static constexpr int HN = ALT ? 128 : 64;                     // keys per softmax warpgroup and tile
  static constexpr int ON = ALT ? D : D / 2;                    // O columns a softmax warpgroup rescales
  static constexpr int EN = D / 2;                              // output columns each softmax warpgroup writes
  static constexpr int SLOT = BN * D * 2;                       // one fp16 K or V tile (32 KB; 16 KB at d = 64)
  // K and V ring slots: at d = 64 the tiles are half as large and both
  // rings twice as deep
  static constexpr int NK = F8 ? 2 : (D == 64 ? 4 : 3), NV = D == 64 ? 4 : 2;
  static constexpr int NSB = 3;                                 // score buffers in TMEM
  static constexpr int Q16_BYTES = BM * D * 2;
  static constexpr int Q8_BYTES = BM * D;
  static constexpr int HALF = BM * 128;                         // one 64-column fp16 slab (128 rows)
  static constexpr int OFF_Q16 = 0;
  static constexpr int OFF_Q8 = OFF_Q16 + Q16_BYTES;
  static constexpr int OFF_QF8 = OFF_Q8 + Q8_BYTES;             // FP8 route only
  static constexpr int OFF_K = OFF_QF8 + (F8 ? Q8_BYTES : 0);
  static constexpr int OFF_V = OFF_K + NK * SLOT;
  static constexpr int OFF_BAR = OFF_V + NV * SLOT;
  static constexpr int OFF_WORDS = OFF_BAR + 256;               // routing words [2 planes][MAXW]
  static constexpr int OFF_SEED = OFF_BAR + 768;                // INT8 accumulator seed blocks (kSeedBytes)
  static constexpr int OFF_XMAX = OFF_BAR + 1280;               // row maxima [2 iterations][2 warpgroups][128],
                                                                // then row sums [2 warpgroups][128]
  static constexpr int OFF_KSC = OFF_XMAX + 3 * 256 * 4;        // key-tile scales of the INT8 route
  static constexpr int MAXJ = 512;                              // key tiles whose scales are staged
  static constexpr int OFF_KSCF8 = OFF_KSC + MAXJ * 4;          // ... of the FP8 route
  static constexpr int BAR_BYTES = 1280 + 3 * 256 * 4 + MAXJ * 4 * (F8 ? 2 : 1);
  static constexpr int MAXW = 64;                               // routing words kept in shared memory
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL = 0;                          // d = 128: one O; DS: O of warpgroup h at 64 h
  static constexpr uint32_t S_COL = 128;                        // + 128 buffer
  static constexpr uint32_t IDESC_S16 = idesc_f16(BM, BN, false);
  static constexpr uint32_t IDESC_S8 = idesc_i8(BM, BN);
  static constexpr uint32_t IDESC_F8 = idesc_f8_e4m3(BM, BN);
  static constexpr uint32_t IDESC_PV = idesc_f16(BM, D, true);
  // INT8 / E4M3 code tiles: one D-byte row per key (128-byte swizzle at
  // d = 128, 64-byte at d = 64)
  static constexpr uint32_t SW8 = (D == 128) ? kSwizzle128 : kSwizzle64;
  static constexpr uint32_t SBO8 = (D == 128) ? 1024u : 512u;
  // 8 softmax warps + K producer, issuer, wait helper, V producer.  The
  // register split is the two-tile kernel's: 2 * 128 * 216 + 128 * 72 = 384 * 168.
  static constexpr int THREADS = 384;
  static constexpr int LAUNCH_REGS = 168, SOFTMAX_REGS = 216, CONTROL_REGS = 72;
  static_assert(2 * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS == THREADS * LAUNCH_REGS,
                "register split must equal the launch allocation");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(D == 64 || D == 128, "head dimension");
  static_assert(!F8 || D == 128, "the FP8 route is built for d = 128");
  static_assert(NK <= 4 && NV <= 4, "ring barriers");
  static_assert(OFF_WORDS + 2 * 4 * MAXW <= OFF_SEED && OFF_SEED + kSeedBytes <= OFF_XMAX, "routing words fit");
};

enum {
  B_QFULL = 0,
  B_SFULL = 1,   // +NSB: S(j) in buffer j mod 3 completed
  B_ODONE = 4,   // +2: P.V(j) completed (barrier j mod 2)
  B_DRAIN = 6,   // every MMA of the CTA completed (one phase)
  B_KFULL = 7,   // +NK (<= 4)
  B_KEMPTY = 11, // +NK
  B_VFULL = 15,  // +NV (<= 4)
  B_VEMPTY = 19, // +NV
  B_PREADY = 23, // +NSB: P(j) of buffer j mod 3 stored (one arrival per softmax warp)
  B_COUNT = 26
};
// Named barriers (0 is __syncthreads):
//   NB_KV:  wait helper (32) <-> issuer (32): operands (and P) ready
//   NB_MAX: the softmax warpgroups (256): row maxima of a tile exchanged
//   NB_EPI: the softmax warpgroups (256): row sums exchanged for the epilogue
// P(j) is signalled on an mbarrier per score buffer, not on a named barrier:
// with S computed up to three tiles ahead the softmax warps can store P(j+1)
// before the issuer has taken P(j), and arrivals of a later round on a named
// barrier would complete an earlier one.  P(j+3), the next phase of P(j)'s
// barrier, needs S(j+3), which is issued only after P.V(j), so each parity
// wait on these barriers is unambiguous.
enum : int { NB_KV = 2, NB_MAX = 3, NB_EPI = 4 };

struct Params3 {
  __half* out;
  int64_t out_st, out_sh;
  const float* q_scales;
  const float* k_scales;
  const uint32_t* bitmask;
  const float* qf8_scales;     // FP8 route: E4M3 tile scales of Q [n_qtiles, Hq] and K [n_ktiles, Hkv]
  const float* kf8_scales;
  const uint32_t* bitmask_f8;  // FP8 route: second bit plane, layout of bitmask
  int64_t mask_hs;
  int W;
  const int32_t* cu;
  const int32_t* cu_k;
  int64_t max_lk;
  int64_t Lq, Lk;
  int Hq, Hkv, g, causal, n_qt_max, batch;
  int kv_chunk;
  float scale_log2;
  DevErr err;
};

__device__ __forceinline__ bool route_bit(const uint32_t* row, int g, int j) {
  if (row == nullptr) return false;
  const int G = j / g;
  return (row[G >> 5] >> (G & 31)) & 1u;
}

// route of key tile j: 0 FP16, 1 INT8 (first bit plane), 2 FP8 (second
// plane, when the first bit is clear)
template <bool F8>
__device__ __forceinline__ int route_of(const uint32_t* row8, const uint32_t* rowf8, int g, int j) {
  if (route_bit(row8, g, j)) return 1;
  if (F8 && route_bit(rowf8, g, j)) return 2;
  return 0;
}

template <int D, int EMU, bool F8>
__global__ void __launch_bounds__(384, 1)
    attn_split_kernel(const __grid_constant__ CUtensorMap tmQ16, const __grid_constant__ CUtensorMap tmQ8,
                      const __grid_constant__ CUtensorMap tmK16, const __grid_constant__ CUtensorMap tmK8,
                      const __grid_constant__ CUtensorMap tmV16, const __grid_constant__ CUtensorMap tmQF8,
                      const __grid_constant__ CUtensorMap tmKF8, const Params3 p) {
  using C = Cfg3<D, F8>;
  constexpr int BN = C::BN, HN = C::HN, ON = C::ON, EN = C::EN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * B_COUNT + 4);
  uint32_t* route_words = reinterpret_cast<uint32_t*>(smem + C::OFF_WORDS);
  float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX);
  float* ksc = reinterpret_cast<float*>(smem + C::OFF_KSC);
  float* kscf8 = reinterpret_cast<float*>(smem + C::OFF_KSCF8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit (query tile I of sequence b, head h).  Grid order: chunk
  // of kv_chunk KV heads (slowest), query tile (heaviest first), sequence,
  // query head within the chunk (fastest), so that the CTAs resident at any
  // time read the K / V of one chunk, sized on the host to stay in L2.
  const int heads_per_chunk = p.kv_chunk * (p.Hq / p.Hkv);
  const int units_per_chunk = heads_per_chunk * p.batch * p.n_qt_max;
  const int chunk = blockIdx.x / units_per_chunk;
  int rest = blockIdx.x - chunk * units_per_chunk;
  const int h = chunk * heads_per_chunk + rest % heads_per_chunk;
  rest /= heads_per_chunk;
  const int b = rest % p.batch;
  const int I = p.n_qt_max - 1 - rest / p.batch;
  const SeqInfo sq = seq_info(p.cu, b, p.Lq, 128);
  const int64_t Lq = sq.len;
  const SeqInfo skq = seq_info(p.cu_k, b, p.Lk, BN);
  const int64_t Lk = p.cu_k ? skq.len : p.Lk;
  const int64_t kstart = p.cu_k ? skq.start : 0;
  if (p.cu_k != nullptr && Lk > p.max_lk) {
    if (threadIdx.x == 0) dev_error(p.err, TM_DEVERR_SEQLEN);
    return;
  }
  if (p.cu != nullptr && I == 0 && threadIdx.x == 0 && Lq > static_cast<int64_t>(p.n_qt_max) * 128)
    dev_error(p.err, TM_DEVERR_SEQLEN);
  const int64_t r0 = static_cast<int64_t>(I) * 128;
  if (r0 >= Lq) return;
  const int rows = static_cast<int>(min(static_cast<int64_t>(128), Lq - r0));
  const int64_t row0 = sq.start + r0;
  const int64_t ig = sq.tile_base + I;
  int nJ = 0;
  if (Lk > 0) {
    int64_t jmax = Lk - 1;
    if (p.causal) jmax = min(jmax, r0 + rows - 1 + Lk - Lq);
    nJ = jmax < 0 ? 0 : static_cast<int>(jmax / BN + 1);
  }
  const uint32_t* mrow = p.bitmask ? p.bitmask + static_cast<int64_t>(h) * p.mask_hs + ig * p.W : nullptr;
  const int hk = h / (p.Hq / p.Hkv);
  const bool words_in_smem = p.W <= C::MAXW;
  const uint32_t* rrow = mrow == nullptr ? nullptr : (words_in_smem ? route_words : mrow);
  const uint32_t* mrowf8 =
      (F8 && p.bitmask_f8) ? p.bitmask_f8 + static_cast<int64_t>(h) * p.mask_hs + ig * p.W : nullptr;
  const uint32_t* rrowf8 = mrowf8 == nullptr ? nullptr : (words_in_smem ? route_words + C::MAXW : mrowf8);

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int i = 0; i < C::NSB; ++i) mbar_init(bar(B_SFULL + i), 1);
    mbar_init(bar(B_ODONE + 0), 1);
    mbar_init(bar(B_ODONE + 1), 1);
    mbar_init(bar(B_DRAIN), 1);
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int i = 0; i < C::NSB; ++i) mbar_init(bar(B_PREADY + i), C::ALT ? 4 : 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 10) {
    seed_blocks_init(reinterpret_cast<uint32_t*>(smem + C::OFF_SEED), lane);
    fence_async_shared();   // generic-proxy stores, read by tcgen05.mma
  }
  if (warp == 8) {
    if (lane == 0) {
      prefetch_tmap(&tmQ16);
      prefetch_tmap(&tmK16);
      prefetch_tmap(&tmV16);
    }
    if (words_in_smem && mrow != nullptr)
      for (int w = lane; w < p.W; w += 32) route_words[w] = __ldg(mrow + w);
    if (words_in_smem && mrowf8 != nullptr)
      for (int w = lane; w < p.W; w += 32) route_words[C::MAXW + w] = __ldg(mrowf8 + w);
    if (mrowf8 != nullptr) {
      const int nst = nJ < C::MAXJ ? nJ : C::MAXJ;
      for (int j = lane; j < nst; j += 32) kscf8[j] = __ldg(p.kf8_scales + (skq.tile_base + j) * p.Hkv + hk);
    }
    // the INT8 route's key-tile scales, so that no softmax step waits on a
    // global load for them
    if (mrow != nullptr) {
      const int nst = nJ < C::MAXJ ? nJ : C::MAXJ;
      for (int j = lane; j < nst; j += 32) ksc[j] = __ldg(p.k_scales + (skq.tile_base + j) * p.Hkv + hk);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_dec<C::CONTROL_REGS>();
    if (warp == 8) {
      // ======================= TMA producers =======================
      // Warp 8 loads Q and then K(j) into K slot j mod 3; warp 11 loads V(j)
      // into V slot j mod 2.  Each waits on its own ring (one thread per
      // warp), so a K tile never queues behind a V slot that a P.V holds.
      if (lane == 0 && nJ > 0) {
        const uint64_t pol_kv = l2_policy_evict_last();
        volatile int never = 0;
        {
          bool any8 = false, anyf8 = false;
          if (mrow != nullptr)
            for (int w = 0; w < p.W; ++w) any8 |= (__ldg(mrow + w) != 0u);
          if (mrowf8 != nullptr)
            for (int w = 0; w < p.W; ++w) anyf8 |= (__ldg(mrowf8 + w) != 0u);
          const uint64_t pol_q = l2_policy_evict_first();
          const int32_t qr = static_cast<int32_t>(row0);
          mbar_arrive_expect_tx(bar(B_QFULL),
                                C::Q16_BYTES + (any8 ? C::Q8_BYTES : 0) + (anyf8 ? C::Q8_BYTES : 0));
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d_hint(sbase + C::OFF_Q16 + hh * C::HALF, &tmQ16, bar(B_QFULL), hh * 64, h, qr, pol_q);
          if (any8) tma_load_3d_hint(sbase + C::OFF_Q8, &tmQ8, bar(B_QFULL), 0, h, qr, pol_q);
          if (anyf8) tma_load_3d_hint(sbase + C::OFF_QF8, &tmQF8, bar(B_QFULL), 0, h, qr, pol_q);
          int nk = 0;
          for (int j = 0; j < nJ; ++j) {
            const int32_t krow = static_cast<int32_t>(kstart + static_cast<int64_t>(j) * BN);
            const int ks = j % C::NK;
            if (j >= C::NK && !mbar_wait(bar(B_KEMPTY + ks), (j / C::NK - 1) & 1, p.err, abort_flag)) break;
            const uint32_t kdst = sbase + C::OFF_K + ks * C::SLOT;
            const int rt = route_of<F8>(rrow, rrowf8, p.g, j);
            if (rt != 0) {   // int8 or E4M3 codes: one 128-byte row per key
              mbar_arrive_expect_tx(bar(B_KFULL + ks), BN * D);
              tma_load_3d_hint(kdst, rt == 1 ? &tmK8 : &tmKF8, bar(B_KFULL + ks), 0, hk, krow, pol_kv);
            } else {
              mbar_arrive_expect_tx(bar(B_KFULL + ks), C::SLOT);
#pragma unroll
              for (int hh = 0; hh < D / 64; ++hh)
                tma_load_3d_hint(kdst + hh * C::HALF, &tmK16, bar(B_KFULL + ks), hh * 64, hk, krow, pol_kv);
            }
            nk = j + 1;
          }
          // Drain: every issued copy has landed before the CTA may exit.
          mbar_wait(bar(B_QFULL), 0, p.err, &never);
          for (int i = (nk > C::NK ? nk - C::NK : 0); i < nk; ++i)
            mbar_wait(bar(B_KFULL + i % C::NK), (i / C::NK) & 1, p.err, &never);
        }
      }
    } else if (warp == 11) {
      if (lane == 0 && nJ > 0) {
        const uint64_t pol_kv = l2_policy_evict_last();
        volatile int never = 0;
        {
          int nv = 0;
          for (int j = 0; j < nJ; ++j) {
            const int32_t krow = static_cast<int32_t>(kstart + static_cast<int64_t>(j) * BN);
            const int vs = j % C::NV;
            if (j >= C::NV && !mbar_wait(bar(B_VEMPTY + vs), (j / C::NV - 1) & 1, p.err, abort_flag)) break;
            const uint32_t vdst = sbase + C::OFF_V + vs * C::SLOT;
            mbar_arrive_expect_tx(bar(B_VFULL + vs), C::SLOT);
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh)
              tma_load_3d_hint(vdst + hh * C::HALF, &tmV16, bar(B_VFULL + vs), hh * 64, hk, krow, pol_kv);
            nv = j + 1;
          }
          for (int i = (nv > C::NV ? nv - C::NV : 0); i < nv; ++i)
            mbar_wait(bar(B_VFULL + i % C::NV), (i / C::NV) & 1, p.err, &never);
        }
      }
    } else if (warp == 9) {
      // ======================= tcgen05 issuer =======================
      // Issue order: S(0), S(1), S(2), then per key tile j: P.V(j), S(j+3).
      // The issuing warp never touches shared memory in its loop except for
      // one routing word per 32 groups (a shared-memory access by the
      // issuing thread delays its next MMA while the MMAs load the port):
      // the wait helper makes every mbarrier wait (operands landed, P
      // stored) and meets it at NB_KV.  Each group of MMAs goes out from one
      // asm statement with its descriptors formed beforehand (mma_f16_ss_n).
      if (nJ > 0) {
        auto kv_handoff = [&]() { named_bar_sync(NB_KV, 64); };
        int wwin = -1;
        uint32_t rw = 0, rwf8 = 0;
        auto route_reg = [&](int j) -> int {
          if (rrow == nullptr && rrowf8 == nullptr) return 0;
          const int G = j / p.g;
          if ((G >> 5) != wwin) {
            wwin = G >> 5;
            rw = rrow != nullptr ? rrow[wwin] : 0u;
            rwf8 = rrowf8 != nullptr ? rrowf8[wwin] : 0u;
          }
          if ((rw >> (G & 31)) & 1u) return 1;
          return (F8 && ((rwf8 >> (G & 31)) & 1u)) ? 2 : 0;
        };
        auto issue_s = [&](int j) {
          const int rt = route_reg(j);
          const bool i8 = rt != 0;   // 8-bit codes: int8 or E4M3
          const int ks = j % C::NK, sb = j % C::NSB;
          const uint32_t kb = sbase + C::OFF_K + ks * C::SLOT;
          const uint32_t d_s = tmem + C::S_COL + 128u * static_cast<uint32_t>(sb);
          if (i8) {
            uint64_t ad[D / 32], bd[D / 32];
            const uint32_t qa = sbase + (rt == 1 ? C::OFF_Q8 : C::OFF_QF8);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
              ad[kk] = smem_desc(qa + kk * 32, 16, C::SBO8, C::SW8);
              bd[kk] = smem_desc(kb + kk * 32, 16, C::SBO8, C::SW8);
            }
            if (elect_one()) {
              if (F8 && rt == 2) {
                mma_f8_ss_n<D / 32>(d_s, ad, bd, C::IDESC_F8, 0u);
              } else {
                const uint64_t sd[3] = {seed_desc(sbase + C::OFF_SEED), seed_desc(sbase + C::OFF_SEED + 128),
                                        seed_desc(sbase + C::OFF_SEED + 256)};
                mma_i8_exact_n<D / 32>(d_s, sd, C::IDESC_S16, ad, bd, C::IDESC_S8);
              }
              tc_commit(bar(B_SFULL + sb));
              tc_commit(bar(B_KEMPTY + ks));
            }
          } else {
            uint64_t ad[D / 16], bd[D / 16];
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::HALF + (kk & 3) * 32;
              ad[kk] = smem_desc(sbase + C::OFF_Q16 + off, 16, 1024, kSwizzle128);
              bd[kk] = smem_desc(kb + off, 16, 1024, kSwizzle128);
            }
            if (elect_one()) {
              mma_f16_ss_n<D / 16>(d_s, ad, bd, C::IDESC_S16, 0u);
              tc_commit(bar(B_SFULL + sb));
              tc_commit(bar(B_KEMPTY + ks));
            }
          }
          __syncwarp();
        };
        auto issue_pv = [&](int j) {
          const int vs = j % C::NV;
          const uint32_t vb = sbase + C::OFF_V + vs * C::SLOT;
          const uint32_t d_s = tmem + C::S_COL + 128u * static_cast<uint32_t>(j % C::NSB);
          uint32_t at[8];
          uint64_t bd[8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // keys 16kk .. 16kk+15: DS / PP, P of the tile's warpgroup in its
            // first 64 columns; otherwise P of warpgroup kk / 4 at its columns
            at[kk] = C::ALT ? d_s + kk * 8 : d_s + (kk >> 2) * HN + (kk & 3) * 8;
            bd[kk] = smem_desc(vb + kk * 2048, C::HALF, 1024, kSwizzle128);
          }
          // DS: P.V(j) accumulates into the O of warpgroup j mod 2, which its
          // first tile (j < 2) initialises
          const uint32_t d_o = tmem + C::O_COL + (C::DS ? static_cast<uint32_t>(D * (j & 1)) : 0u);
          const uint32_t acc = (C::DS ? j > 1 : j > 0) ? 1u : 0u;
          tc_fence_after();   // orders the softmax warps' TMEM stores of P before the MMAs read it
          if (elect_one()) {
            mma_f16_ts_n<8>(d_o, at, bd, C::IDESC_PV, acc);
            tc_commit(bar(B_ODONE + (j & 1)));
            tc_commit(bar(B_VEMPTY + vs));
          }
          __syncwarp();
        };
        TM_TRACE_DECL
        // trace events (TM_TRACE builds): recorded by lane 0, then the warp
        // reconverges before its next aligned barrier
        auto trace_ev = [&](int ev) {
          if (lane == 0) TM_TRACE_EV(3, ev);
          __syncwarp();
        };
        kv_handoff();   // Q landed
        for (int j = 0; j < C::NSB && j < nJ; ++j) {
          kv_handoff();   // K(j)
          issue_s(j);
        }
        for (int j = 0; j < nJ; ++j) {
          kv_handoff();   // V(j) landed and P(j) stored
          trace_ev(20);
          issue_pv(j);
          trace_ev(21);
          if (j + C::NSB < nJ) {
            kv_handoff();   // K(j+3)
            trace_ev(22);
            issue_s(j + C::NSB);
            trace_ev(24);
          }
        }
        if (elect_one()) tc_commit(bar(B_DRAIN));
        __syncwarp();
        if (lane == 0) {
          volatile int never = 0;
          mbar_wait(bar(B_DRAIN), 0, p.err, &never);
        }
        __syncwarp();
      }
    } else if (warp == 10) {
      // ======================= wait helper =======================
      // Makes the issuer's operand waits in the issuer's order and meets it
      // at NB_KV after each.  A wait that times out or sees the abort flag
      // only records the failure; every handoff is still taken.
      if (nJ > 0) {
        auto wait1 = [&](uint32_t bb, uint32_t par) {
          if (lane == 0) mbar_wait(bb, par, p.err, abort_flag);
        };
        auto handoff = [&]() {
          __syncwarp();
          named_bar_sync(NB_KV, 64);
        };
        auto wait_k = [&](int j) { wait1(bar(B_KFULL + j % C::NK), (j / C::NK) & 1); };
        wait1(bar(B_QFULL), 0);
        handoff();
        for (int j = 0; j < C::NSB && j < nJ; ++j) {
          wait_k(j);
          handoff();
        }
        for (int j = 0; j < nJ; ++j) {
          wait1(bar(B_VFULL + j % C::NV), (j / C::NV) & 1);
          wait1(bar(B_PREADY + j % C::NSB), (j / C::NSB) & 1);
          handoff();
          if (j + C::NSB < nJ) {
            wait_k(j + C::NSB);
            handoff();
          }
        }
      }
    }
  } else {
    // ======================= softmax (warpgroup hw = keys [64 hw, 64 hw + 64)) =======================
    regs_inc<C::SOFTMAX_REGS>();
    const int hw = warp >> 2;
    const int r = threadIdx.x & 127;                 // row in the tile = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // the O columns this warpgroup rescales: its own O (DS), all of O (PP),
    // or its half of O's columns
    const uint32_t o_addr = lane_addr + C::O_COL + (C::PP ? 0u : static_cast<uint32_t>(ON * hw));
    float* mpub = xmax;   // PP: reference max of the last stored tile, per row
    const bool row_ok = r < rows;
    const int64_t i_row = r0 + r;
    int64_t lim = -1;
    if (row_ok) lim = p.causal ? min(Lk - 1, i_row + Lk - Lq) : Lk - 1;
    float c8_row = 0.f, cf8_row = 0.f;
    if (mrow != nullptr) c8_row = __ldg(p.q_scales + ig * p.Hq + h) * p.scale_log2;
    if (mrowf8 != nullptr) cf8_row = __ldg(p.qf8_scales + ig * p.Hq + h) * p.scale_log2;
    const SeqInfo sk = seq_info(p.cu_k, b, p.Lk, BN);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    TM3_PH_DECL
    // DS / PP: this warpgroup's key tiles are j = hw, hw + 2, ...; otherwise
    // every key tile, keys [64 hw, 64 hw + 64)
    const int key_off = C::ALT ? 0 : HN * hw;
    for (int j = C::ALT ? hw : 0; j < nJ; j += C::ALT ? 2 : 1) {
      const int sb = j % C::NSB;
      const uint32_t s_addr = lane_addr + C::S_COL + 128u * sb + key_off;
      const int rt = route_of<F8>(rrow, rrowf8, p.g, j);
      const bool i8 = rt == 1;   // INT8 and FP8 scores arrive in fp32 (see mma_i8_exact_n)
      float c = p.scale_log2;
      if (i8) {
        const float ks = j < C::MAXJ ? ksc[j] : __ldg(p.k_scales + (sk.tile_base + j) * p.Hkv + hk);
        c = fmaxf(c8_row * ks, 1e-30f);
      } else if (F8 && rt == 2) {
        const float ks = j < C::MAXJ ? kscf8[j] : __ldg(p.kf8_scales + (sk.tile_base + j) * p.Hkv + hk);
        c = fmaxf(cf8_row * ks, 1e-30f);
      }
      // No early exit: the issuer expects one P handoff per key tile.
      if (!mbar_wait(bar(B_SFULL + sb), (j / C::NSB) & 1, p.err, abort_flag)) ok = false;
      tc_fence_after();
      __syncwarp();
      TM3_PH(0);
      float x[HN];
      {
        uint32_t u[HN];
#pragma unroll
        for (int cc = 0; cc < HN / 32; ++cc) tmem_ld32p(s_addr + cc * 32, u + cc * 32);
        tmem_wait_ld_regs<HN>(u);
#pragma unroll
        for (int e = 0; e < HN; ++e) x[e] = __uint_as_float(u[e]);
      }
      TM3_PH(1);
      const int64_t nv64 = lim - (static_cast<int64_t>(j) * BN + key_off) + 1;
      const int nv = nv64 <= 0 ? 0 : (nv64 >= HN ? HN : static_cast<int>(nv64));
      if (!__all_sync(0xffffffffu, nv == HN)) {
#pragma unroll
        for (int e = 0; e < HN; ++e) x[e] = (e < nv) ? x[e] : -INFINITY;
      }
      // row max of the tile in log2 units (-inf when no key is visible); with
      // the keys split between the warpgroups, over both halves
      {
        float mt;
        if constexpr (C::ALT) {
          mt = row_max<HN>(x) * c;
        } else {
          float* xm = xmax + (j & 1) * 256;
          xm[hw * 128 + r] = row_max<HN>(x) * c;   // -inf when no key of this half is visible
          __syncwarp();
          named_bar_sync(NB_MAX, 256);
          mt = fmaxf(xm[r], xm[128 + r]);
        }
        // m_prev: the reference the previous tile of this stream used.  PP:
        // the previous tile (j-1) belongs to the other warpgroup; wait until
        // its P is stored (it published its reference before signalling).
        // The barrier's next phase, P(j+2), is this warpgroup's own and its
        // previous one, P(j-4), completed before S(j) could be issued, so
        // the parity wait is unambiguous.
        float m_prev = m_used;
        if constexpr (C::PP) {
          m_prev = -INFINITY;
          if (j > 0) {
            const int jq = j - 1;
            if (!mbar_wait(bar(B_PREADY + jq % C::NSB), (jq / C::NSB) & 1, p.err, abort_flag)) ok = false;
            m_prev = mpub[r];
          }
        }
        float alpha = 1.f;   // O's factor
        float m_new = m_prev;
        if (mt > m_prev + kLazyRescaleLog2) {
          alpha = ex2_approx(m_prev - mt);
          m_new = mt;
        }
        // this warpgroup's row sum was accumulated against m_used (PP: the
        // reference of its own previous tile, which the other stream's tile
        // may have raised since)
        float alpha_l = alpha;
        if constexpr (C::PP) alpha_l = (m_used == m_new) ? 1.f : ex2_approx(m_used - m_new);
        m_used = m_new;
        if constexpr (C::PP) mpub[r] = m_new;   // read by the other warpgroup once P(j) is signalled
                TM3_PH(2);
        const float msub = (m_used == -INFINITY) ? 0.f : m_used;
        const uint64_t c2 = f2pack(c, c);
        const uint64_t nm2 = f2pack(-msub, -msub);
        uint32_t pk[HN / 2];
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int e = 0; e < HN; e += 2) {
          const uint64_t y2 = f2fma(f2pack(x[e], x[e + 1]), c2, nm2);
          float p0, p1;
          if (EMU > 0 && ((e >> 1) & 7) < EMU) {
            exp2_poly2(y2, p0, p1);
          } else {
            float y0, y1;
            f2unpack(y2, y0, y1);
            p0 = ex2_approx(y0);
            p1 = ex2_approx(y1);
          }
          acc2[(e >> 1) & 3] = f2add(acc2[(e >> 1) & 3], f2pack(p0, p1));
          pk[e >> 1] = pack_half2(p0, p1);
          // PP: each 32 columns of P go to TMEM as soon as they are complete
          // (their scores were read into registers already), so that fewer
          // registers stay live through the loop
          if (C::PP && (e & 63) == 62) {
            __syncwarp();
            tmem_st32p(s_addr + (e >> 6) * 32, pk + (e >> 6) * 32);
          }
        }
        {
          const uint64_t s2 = f2add(f2add(acc2[0], acc2[1]), f2add(acc2[2], acc2[3]));
          float s0, s1;
          f2unpack(s2, s0, s1);
          l = l * alpha_l + (s0 + s1);
        }
        TM3_PH(3);
        __syncwarp();
        // P_hw(j) over the first HN / 2 columns of this warpgroup's scores
        if constexpr (!C::PP) {
#pragma unroll
          for (int cc = 0; cc < HN / 64; ++cc) tmem_st32p(s_addr + cc * 32, pk + cc * 32);
        }
        // This warpgroup's O columns are rescaled only when a row of this warp
        // raised the running max.  Then the previous P.V into them, P.V(jp)
        // with jp = j - 2 (DS) or j - 1 (PP and the split keys), must have
        // completed.  It commits to
        // barrier jp mod 2, whose phases are P.V(jp mod 2), P.V(jp mod 2 + 2),
        // ...  S(j) was issued after P.V(j-3) and has completed, so P.V(jp-2)
        // is done; P.V(jp+2) cannot be, as the issuer takes P(jp+2) (DS: P(j);
        // otherwise P(j+1)) only after this warpgroup signals it at the end of
        // this step or a later one: the parity wait is unambiguous.
        const int jp = j - (C::DS ? 2 : 1);
        if (jp >= 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!mbar_wait(bar(B_ODONE + (jp & 1)), (jp >> 1) & 1, p.err, abort_flag)) ok = false;
          tc_fence_after();
          __syncwarp();
          const uint64_t a2 = f2pack(alpha, alpha);
          // 64 columns at a time (PP rescales all 128 of O)
#pragma unroll
          for (int oc = 0; oc < ON; oc += 64) {
            uint32_t o[64];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) tmem_ld32p(o_addr + oc + cc * 32, o + cc * 32);
            tmem_wait_ld_regs<64>(o);
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              float o0, o1;
              f2unpack(f2mul(f2pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), o0, o1);
              o[e] = __float_as_uint(o0);
              o[e + 1] = __float_as_uint(o1);
            }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) tmem_st32p(o_addr + oc + cc * 32, o + cc * 32);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      TM3_PH(4);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PREADY + sb));   // this warp's rows of P(j) stored
      TM3_PH(5);
    }
#ifdef TM_PHASES
    if ((threadIdx.x & 127) == 0 && blockIdx.x == g_tm_trace_block) {
      for (int i = 0; i < 6; ++i) g_tm_trace[hw][TM_TRACE_EVENTS - 8 + i] = static_cast<unsigned long long>(tm_ph[i]);
      g_tm_trace[hw][TM_TRACE_EVENTS - 2] = static_cast<unsigned long long>(nJ);
    }
    __syncwarp();
#endif
    // ---- epilogue: row sums over both warpgroups (DS / PP: with each
    // warpgroup's reference max), then this warpgroup's EN output columns
    bool have_o = false;
    if (ok && nJ > 0) {
      have_o = mbar_wait(bar(B_DRAIN), 0, p.err, abort_flag);
      tc_fence_after();
    }
    float* xs = xmax + 512;   // past both iterations' maxima
    float* xm_epi = xmax + (C::PP ? 256 : 0);   // PP: clear of the published maxima
    xs[hw * 128 + r] = l;
    if constexpr (C::ALT) xm_epi[hw * 128 + r] = m_used;
    __syncwarp();
    named_bar_sync(NB_EPI, 256);
    // DS: stream w contributes a_w * O_w and a_w * l_w with a_w = 2^(m_w - m),
    // m the larger running max; a stream without a visible key (m_w = -inf)
    // contributes nothing.  PP: O already holds every tile against the last
    // tile's reference m (the larger of the two); each warpgroup's row sum
    // l_w is against the reference of its own last tile, so it enters as
    // a_w * l_w alike.
    float a0 = 1.f, a1 = 0.f, inv;
    if constexpr (C::ALT) {
      const float m0 = xm_epi[r], m1 = xm_epi[128 + r];
      const float mm = fmaxf(m0, m1);
      a0 = m0 == -INFINITY ? 0.f : (m0 == mm ? 1.f : ex2_approx(m0 - mm));
      a1 = m1 == -INFINITY ? 0.f : (m1 == mm ? 1.f : ex2_approx(m1 - mm));
      const float lsum = xs[r] * a0 + xs[128 + r] * a1;
      inv = (mm != -INFINITY && lsum > 0.f) ? 1.f / lsum : 0.f;
    } else {
      const float lsum = xs[r] + xs[128 + r];
      inv = (m_used != -INFINITY && lsum > 0.f) ? 1.f / lsum : 0.f;
    }
    __syncwarp();
    const uint32_t e_addr = lane_addr + C::O_COL + EN * hw;
    uint32_t o[EN];
    if (__all_sync(0xffffffffu, have_o)) {
#pragma unroll
      for (int cc = 0; cc < EN / 32; ++cc) tmem_ld32p(e_addr + cc * 32, o + cc * 32);
      if constexpr (C::DS) {
        // the same columns of stream 1's O (written only when nJ > 1)
        uint32_t o1[EN];
        if (nJ > 1) {
#pragma unroll
          for (int cc = 0; cc < EN / 32; ++cc) tmem_ld32p(e_addr + D + cc * 32, o1 + cc * 32);
          tmem_wait_ld_regs<EN>(o1);
        } else {
#pragma unroll
          for (int e = 0; e < EN; ++e) o1[e] = 0u;
        }
        tmem_wait_ld_regs<EN>(o);
#pragma unroll
        for (int e = 0; e < EN; ++e)
          o[e] = __float_as_uint(__uint_as_float(o[e]) * a0 + __uint_as_float(o1[e]) * a1);
      } else {
        tmem_wait_ld_regs<EN>(o);
      }
    } else {
#pragma unroll
      for (int e = 0; e < EN; ++e) o[e] = 0u;
    }
    if (row_ok) {
      __half* orow = p.out + (row0 + r) * p.out_st + static_cast<int64_t>(h) * p.out_sh + EN * hw;
#pragma unroll
      for (int cc = 0; cc < EN / 8; ++cc) {
        uint4 pkt;
        pkt.x = pack_half2(__uint_as_float(o[8 * cc + 0]) * inv, __uint_as_float(o[8 * cc + 1]) * inv);
        pkt.y = pack_half2(__uint_as_float(o[8 * cc + 2]) * inv, __uint_as_float(o[8 * cc + 3]) * inv);
        pkt.z = pack_half2(__uint_as_float(o[8 * cc + 4]) * inv, __uint_as_float(o[8 * cc + 5]) * inv);
        pkt.w = pack_half2(__uint_as_float(o[8 * cc + 6]) * inv, __uint_as_float(o[8 * cc + 7]) * inv);
        st_global_stream_v4(reinterpret_cast<uint4*>(orow) + cc, pkt);
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

#ifndef TM_EXP2_EMU_PAIRS
#define TM_EXP2_EMU_PAIRS 3       // exp2 pairs (of every 8) evaluated on the FMA pipe
#endif
// At d = 64 (dual stream) the FMA pipe also carries both streams' row sums
// and packing with half the MMA time per tile to hide them: 2 of 8 pairs on
// the FMA pipe measured 1-3 % faster than 3 on the MLX-shaped d = 64 runs and
// on a routed L = 16384 launch, 4 of 8 5 % slower.
#ifndef TM_EXP2_EMU_PAIRS_D64
#define TM_EXP2_EMU_PAIRS_D64 2
#endif
template <int D>
constexpr int kEmuPairs = D == 64 ? TM_EXP2_EMU_PAIRS_D64 : TM_EXP2_EMU_PAIRS;

std::mutex g_mu3;

// One-time kernel attributes; the warpgroup register split assumes exactly
// LAUNCH_REGS per thread at launch, so a build that differs is refused.
template <int D, bool F8>
tm_status prepare_split_kernel() {
  static bool attr_done = false;
  std::lock_guard<std::mutex> lk(g_mu3);
  if (attr_done) return TM_OK;
  auto kern = attn_split_kernel<D, kEmuPairs<D>, F8>;
  cudaFuncAttributes fa;
  tm_status st = check_cuda(cudaFuncGetAttributes(&fa, kern));
  if (st != TM_OK) return st;
  if (fa.numRegs != Cfg3<D, F8>::LAUNCH_REGS) return TM_ERR_UNSUPPORTED;
  st = check_cuda(
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg3<D, F8>::SMEM_BYTES));
  if (st != TM_OK) return st;
  attr_done = true;
  return TM_OK;
}

template <int D>
tm_status launch_split(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                       const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                       const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                       cudaStream_t stream, const Fp8Route* f8) {
  const bool use_f8 = D == 128 && f8 != nullptr && f8->bitmask != nullptr;
  tm_status st = use_f8 ? prepare_split_kernel<128, true>() : prepare_split_kernel<D, false>();
  if (st != TM_OK) return st;
  CUtensorMap mQ16, mQ8, mK16, mK8, mV16, mQF8, mKF8;
  st = encode_thd_map(&mQ16, q->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, q->T, q->H, D, q->stride_t,
                      q->stride_h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mK16, k->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, k->T, k->H, D, k->stride_t,
                      k->stride_h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mV16, v->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, v->T, v->H, D, v->stride_t,
                      v->stride_h, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  const CUtensorMapSwizzle swz8 = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (bitmask != nullptr) {
    st = encode_thd_map(&mQ8, q->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->T, q->H, D, q->H * D, D, D, 128,
                        swz8);
    if (st != TM_OK) return st;
    st = encode_thd_map(&mK8, k->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k->T, k->H, D, k->H * D, D, D, 128,
                        swz8);
    if (st != TM_OK) return st;
  } else {
    mQ8 = mQ16;
    mK8 = mK16;
  }
  if (use_f8) {
    st = encode_thd_map(&mQF8, f8->q_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->T, q->H, D, q->H * D, D, D, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TM_OK) return st;
    st = encode_thd_map(&mKF8, f8->k_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k->T, k->H, D, k->H * D, D, D, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TM_OK) return st;
  } else {
    mQF8 = mQ8;
    mKF8 = mK8;
  }
  Params3 p;
  p.out = static_cast<__half*>(out->data);
  p.out_st = out->stride_t;
  p.out_sh = out->stride_h;
  p.q_scales = static_cast<const float*>(q->scales);
  p.k_scales = static_cast<const float*>(k->scales);
  p.bitmask = bitmask;
  p.qf8_scales = use_f8 ? f8->q_scales : nullptr;
  p.kf8_scales = use_f8 ? f8->k_scales : nullptr;
  p.bitmask_f8 = use_f8 ? f8->bitmask : nullptr;
  p.mask_hs = mask_hs;
  p.cu = cu;
  p.cu_k = cu ? (cu_k ? cu_k : cu) : nullptr;
  p.Lq = q->T;
  p.Lk = k->T;
  p.Hq = static_cast<int>(q->H);
  p.Hkv = static_cast<int>(k->H);
  p.g = g;
  p.causal = causal ? 1 : 0;
  p.batch = cu ? batch : 1;
  const int64_t maxq = cu ? max_q : q->T;
  const int64_t maxk = cu ? max_k : k->T;
  p.max_lk = maxk;
  p.n_qt_max = static_cast<int>((maxq + 127) / 128);
  p.W = tm_mask_words(maxk, 128, g);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(D)));
  p.err = DevErr{device_error_word()};
  // KV heads per scheduling chunk: as many as keep their K / V (fp16 K, int8
  // K, fp16 V) within ~40 MB of L2, widened until a chunk fills two waves of
  // 148 CTAs; always a divisor of Hkv.
  {
    const double kv_bytes = static_cast<double>(maxk) * D * (2 + 1 + 2);
    int c = static_cast<int>(40.0e6 / (kv_bytes > 1.0 ? kv_bytes : 1.0));
    c = c < 1 ? 1 : (c > p.Hkv ? p.Hkv : c);
    while (c < p.Hkv && static_cast<int64_t>(c) * (p.Hq / p.Hkv) * p.batch * p.n_qt_max < 2 * 148) ++c;
    while (p.Hkv % c) ++c;
    p.kv_chunk = c;
  }
  const int64_t grid = static_cast<int64_t>(p.n_qt_max) * p.batch * p.Hq;
  if (grid == 0) return TM_OK;
  if (grid > 0x7fffffffLL) return TM_ERR_UNSUPPORTED;
  if (use_f8)
    attn_split_kernel<128, kEmuPairs<128>, true><<<static_cast<unsigned>(grid), Cfg3<128, true>::THREADS,
                                                      Cfg3<128, true>::SMEM_BYTES, stream>>>(
        mQ16, mQ8, mK16, mK8, mV16, mQF8, mKF8, p);
  else
    attn_split_kernel<D, kEmuPairs<D>, false><<<static_cast<unsigned>(grid), Cfg3<D, false>::THREADS,
                                                    Cfg3<D, false>::SMEM_BYTES, stream>>>(
        mQ16, mQ8, mK16, mK8, mV16, mQF8, mKF8, p);
  return check_cuda(cudaGetLastError());
}

}  // namespace

tm_status launch_attn_split(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                            cudaStream_t stream, const Fp8Route* f8) {
  const bool use_f8 = f8 != nullptr && f8->bitmask != nullptr;
  if (q->d == 128)
    return launch_split<128>(q, k, v, out, cu, cu_k, batch, max_q, max_k, bitmask, mask_hs, g, causal, stream, f8);
  if (q->d == 64 && !use_f8)
    return launch_split<64>(q, k, v, out, cu, cu_k, batch, max_q, max_k, bitmask, mask_hs, g, causal, stream, f8);
  return TM_ERR_UNSUPPORTED;
}

}  // namespace tmk
