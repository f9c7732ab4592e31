// tm_attn2.cu -- fused tile-routed attention, two 128-row query tiles per CTA.
//
// TileMix (Lattice paper page), abstract: score tiles routed per group of g
// key tiles to an FP16 or an INT8 QK^T, both feeding one online-softmax state.
// This is the production layout for 128 x 128 score tiles.  On B200 the
// softmax (one exp2 per score, plus max / sum / conversion) costs about as
// much as the FP16 MMAs of a tile, so the kernel is built to keep the tensor
// pipe and the softmax warps busy at the same time:
//
//   * one CTA owns query tiles A = 2P and B = 2P+1 of one head; its two
//     softmax warpgroups (warps 0-3 on tile A, warps 4-7 on tile B) alternate
//     on the tensor core: while one warpgroup computes exp2 on its score
//     tile, the tensor pipe runs the other tile's P.V and next QK^T;
//   * TMEM holds S_A, S_B (128 columns each; P overwrites S in place as fp16)
//     and the fp32 accumulators O_A, O_B;
//   * an INT8-routed score tile leaves the tensor core as exact fp32 numbers
//     (mma_i8_exact_n: a seed MMA, the kind::i8 MMAs, an unseed MMA), so the
//     softmax handles both routes alike, only the scale differs; the INT8
//     QK^T takes 6 MMAs of M128 N128 against the FP16 route's 8;
//   * K / V arrive through a ring of tile-sized shared-memory slots: per key
//     tile the producer loads the fp16 K tile if either query tile routes it
//     FP16, the int8 K-code tile if either routes it INT8 (both when they
//     differ), and the fp16 V tile; slots are released by tcgen05.commit once
//     the MMAs reading them have completed;
//   * the softmax arithmetic runs on packed fp32 pairs (f32x2 FMA / ADD),
//     and 3 of every 8 exp2 pairs run as a degree-3 minimax polynomial on the
//     FMA pipe (Cody-Waite split 2^y = 2^n * 2^f, f in [-1/2, 1/2];
//     coefficients fitted by the Remez exchange, max relative error 7.5e-5,
//     below the fp16 rounding of P), the rest on MUFU.ex2, so that neither
//     the MUFU pipe nor instruction issue alone bounds the softmax;
//   * K / V loads carry an evict-last L2 policy and Q an evict-first one,
//     and the output is written with streaming stores;
//   * chunked mode (template argument CH; all-FP16 rows of 64 key tiles or
//     more): each tile's 128 score columns hold two 64-key chunks, and the
//     QK^T of chunk c+2 follows the P.V of chunk c into the same half, so
//     the tensor pipe computes the next chunk's scores while the softmax
//     works on the current one.
// Every mbarrier wait is bounded (tm_device.cuh).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tm_attn_internal.h"
#include "tm_device.cuh"
#include "tm_host.h"

#if defined(TM_TRACE) || defined(TM_TIMEOUT_INFO)
extern "C" int tm_debug_timeout_read(unsigned int* host) {
  if (cudaMemcpyFromSymbol(host, tmk::g_tm_timeout_info, sizeof(tmk::g_tm_timeout_info)) != cudaSuccess) return -1;
  static const unsigned int zero[5] = {0, 0, 0, 0, 0};
  return cudaMemcpyToSymbol(tmk::g_tm_timeout_info, zero, sizeof(zero)) == cudaSuccess ? 0 : -1;
}
#endif
#ifdef TM_TRACE
extern "C" int tm_debug_trace_read(unsigned long long* host, unsigned int block) {
  if (host == nullptr) {
    static unsigned long long zero[TM_TRACE_ROLES][TM_TRACE_EVENTS];
    if (cudaMemcpyToSymbol(g_tm_trace, zero, sizeof(zero)) != cudaSuccess) return -1;
    return cudaMemcpyToSymbol(g_tm_trace_block, &block, sizeof(block)) == cudaSuccess ? 0 : -1;
  }
  return cudaMemcpyFromSymbol(host, g_tm_trace, sizeof(g_tm_trace)) == cudaSuccess ? 0 : -1;
}
#endif


// Softmax phase profile (compiled only with TM_PHASES, together with
// TM_TRACE): the tracing thread sums SM-clock deltas per phase in registers
// and stores the sums once, so the profile costs a few cycles per phase.
#ifdef TM_PHASES
#define TM_SM_EV(ev) do { } while (0)
#define TM_PH_DECL long long tm_ph[8] = {0, 0, 0, 0, 0, 0, 0, 0}; long long tm_ph_t = clock64();
#define TM_PH(i) do { const long long tm_now = clock64(); tm_ph[i] += tm_now - tm_ph_t; tm_ph_t = tm_now; } while (0)
#else
#define TM_SM_EV(ev) do { if (tracer) TM_TRACE_EV(t, ev); } while (0)
#define TM_PH_DECL
#define TM_PH(i) do { } while (0)
#endif

namespace tmk {
namespace {

// trace event ids (roles: 0 = softmax A, 1 = softmax B, 2 = producer, 3 = issuer)
enum : unsigned {
  EV_S_READY = 1, EV_EXP_DONE = 2, EV_O_READY = 3, EV_RESCALED = 4, EV_P_RELEASED = 5, EV_EPI_DONE = 6,
  EV_ACQUIRED = 10, EV_K_READY = 20, EV_PV_A = 21, EV_S_A = 22, EV_PV_B = 23, EV_S_B = 24, EV_V_READY = 25,
  EV_START = 30, EV_KWAIT_BEGIN = 31, EV_KWAIT_END = 32, EV_VWAIT_BEGIN = 33, EV_SLOADED = 7, EV_MAXED = 8,
  EV_P_SEEN = 26, EV_MMA_ISSUED = 27, EV_HW_KV_BEGIN = 40, EV_HW_KV_END = 41, EV_HW_P_BEGIN = 42,
  EV_HW_P_END = 43
};

// CACHE: K / V come from an INT8 cache (codes + fp16 scale per token and KV
// head): a dequantisation warpgroup (warps 12-15) writes the fp16 K tiles of
// FP16-routed key tiles and every fp16 V tile into the ring, the producer
// brings the int8 K code tiles of INT8-routed ones, and the softmax applies
// the per-token key scales of INT8 tiles per column.
template <int D, bool CACHE = false, bool TOKS = false>
struct Cfg2 {
  static constexpr int BM = 128, BN = 128;
  static constexpr int SLOT = BN * D * 2;                // one fp16 K or V tile
  static constexpr int NSLOT = 131072 / SLOT;            // 4 (d=128) or 8 (d=64)
  static constexpr int Q16_BYTES = BM * D * 2;           // per query tile
  static constexpr int Q8_BYTES = BM * D;
  static constexpr int HALF = BM * 128;                  // one 64-column fp16 slab (128 rows)
  static constexpr int OFF_Q16 = 0;
  static constexpr int OFF_Q8 = 2 * Q16_BYTES;
  static constexpr int OFF_SLOT = OFF_Q8 + 2 * Q8_BYTES;
  static constexpr int OFF_BAR = OFF_SLOT + NSLOT * SLOT;
  static constexpr int BAR_BYTES = 2048;                 // barriers, routing words, seed blocks, key-tile scales
  // Without CACHE: routing words [2][64] at +256, seed blocks at +768,
  // INT8 key-tile scales at +1152.  With CACHE: routing words [2][32] at
  // +256, the extra barriers at +512, seed blocks at +640, two stages of
  // per-token key scales (128 fp32 each) at +1024.
  static constexpr int OFF_SEED = OFF_BAR + (CACHE ? 640 : (TOKS ? 512 : 768));   // INT8 accumulator seed blocks
  static constexpr int OFF_KSC = OFF_BAR + 1152;
  static constexpr int KSC_MAX = CACHE ? 0 : 224;        // key tiles whose INT8 scales are staged
  static constexpr int OFF_CBAR = OFF_BAR + 512;         // CACHE: key-scale stage barriers
  static constexpr int OFF_KST = OFF_BAR + 1024;         // CACHE: key-scale stages [2][128] fp32
  static constexpr int MAXW = (CACHE || TOKS) ? 32 : 64;  // routing words per query tile kept in smem
  // TOKS (per-token key scales; fp16 K / V): routing words [2][32] at +256,
  // seed blocks at +512, and one row of 128 fp32 key scales per softmax
  // warpgroup at +896, which that warpgroup writes and reads.
  static constexpr int OFF_KSTT = OFF_BAR + 896;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S16 = idesc_f16(BM, BN, false);
  static constexpr uint32_t IDESC_S8 = idesc_i8(BM, BN);
  static constexpr uint32_t IDESC_F8 = idesc_f8_e4m3(BM, BN);           // the FP8 route (F8 launches)
  static constexpr uint32_t IDESC_S16_64 = idesc_f16(BM, 64, false);   // chunked mode: 64-key chunks
  static constexpr uint32_t IDESC_S8_64 = idesc_i8(BM, 64);
  static constexpr uint32_t IDESC_PV = idesc_f16(BM, D, true);
  static constexpr uint32_t SW8 = (D == 128) ? kSwizzle128 : kSwizzle64;
  static constexpr uint32_t SBO8 = (D == 128) ? 1024u : 512u;
  // 8 softmax warps + (producer, MMA issuers, wait helper) warps, and with
  // CACHE the 4 dequantisation warps.  Launch: 168 registers per thread (3
  // warps per SM sub-partition); the softmax warpgroups then take 216 and the
  // control warpgroup keeps 72: 2 * 128 * 216 + 128 * 72 = 384 * 168.  With
  // CACHE: 128 at launch (4 warps per sub-partition), softmax 208, control
  // 48, dequantisation 48: 2 * 128 * 208 + 128 * 48 + 128 * 48 = 512 * 128.
  // TOKS: softmax 224 (its per-column key-scale multiply), control 56:
  // 2 * 128 * 224 + 128 * 56 = 384 * 168.
  static constexpr int THREADS = CACHE ? 512 : 384;
  static constexpr int LAUNCH_REGS = CACHE ? 128 : 168, SOFTMAX_REGS = CACHE ? 208 : (TOKS ? 224 : 216);
  static constexpr int CONTROL_REGS = CACHE ? 48 : (TOKS ? 56 : 72), DEQ_REGS = CACHE ? 48 : 0;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(CACHE ? (OFF_BAR + 256 + 4 * 2 * MAXW <= OFF_CBAR && OFF_CBAR + 8 * 10 <= OFF_SEED &&
                         OFF_SEED + kSeedBytes <= OFF_KST &&
                         OFF_KST + 2 * 128 * 4 <= OFF_BAR + BAR_BYTES)
                      : (OFF_SEED + kSeedBytes <= OFF_KSC && OFF_KSC + 4 * KSC_MAX <= OFF_BAR + BAR_BYTES),
                "layout");
  static_assert(!TOKS || (OFF_BAR + 256 + 4 * 2 * MAXW <= OFF_SEED && OFF_SEED + kSeedBytes <= OFF_KSTT &&
                          OFF_KSTT + 2 * 512 <= OFF_BAR + BAR_BYTES),
                "per-token key-scale rows");
  static_assert(2 * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS + 128 * DEQ_REGS == THREADS * LAUNCH_REGS,
                "register split must equal the launch allocation");
  __host__ __device__ static constexpr uint32_t s_col(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t o_col(int t) { return 256u + D * t; }
};

enum {
  C_QFULL = 0,
  C_SFULL = 1,   // +2 (tile A, B)
  C_ODONE = 3,   // +2
  C_DRAIN = 5,   // +2 (one per issuer)
  C_PFULL = 7,   // +2: P_t stored (single-issuer mode; count 128)
  C_FULL = 9,    // +NSLOT (<= 8)
  C_EMPTY = 17,  // +NSLOT; one release per issuer that reads the slot's tiles
  C_SFULL2 = 25, // +4 (chunked mode: 2 tiles x 2 score slots)
  C_COUNT = 29
};
// Named barriers (0 is __syncthreads):
//   NB_P + t:  softmax warpgroup t (128, arrive) -> issuer t (32, sync): P_t stored
//   NB_KV + t: wait helper (32) <-> issuer t (32): operands landed
//   NB_START: softmax A (128, arrive) -> issuer B (32, sync), once: P_A(0) stored
//   NB_DEQ:    the four dequantisation warps (128, CACHE): a tile is written
//   NB_KST + t: softmax warpgroup t (128, TOKS): its key-scale row written / read
enum : int { NB_P = 1, NB_KV = 3, NB_START = 5, NB_DEQ = 6, NB_KST = 7 };
// CACHE barriers (at OFF_CBAR): key-scale stage s written (count 128), and
// read by query tile t (count 4: one arrival per softmax warp); the code
// tile of a ring slot's next fp16 tile landed (count 1, TMA bytes).
enum { CB_KSFULL = 0, CB_KSEMPTY = 2, CB_CFULL = 6, CB_COUNT = 10 };

struct Params2 {
  __half* out;
  int64_t out_st, out_sh;
  const float* q_scales;
  const float* k_scales;
  const uint32_t* bitmask;
  int64_t mask_hs;
  int W;
  const int32_t* cu;
  const int32_t* cu_k;   // key offsets (= cu unless separate)
  int64_t max_lk;        // longest key row the launch was sized for
  int64_t Lq, Lk;
  int Hq, Hkv, g, causal, n_pair_max, n_qt_max, batch;
  int kv_chunk;            // KV heads per scheduling chunk (divides Hkv)
  float scale_log2;
  DevErr err;
  int sched_zero;        // always 0 (see its use in the softmax)
  // CACHE: fp16 scales [T, Hkv] of the K and V cache (the codes come by TMA)
  const __half* k_tok_scale;
  const __half* v_tok_scale;
  // TOKS: per-token K scales laid out [Hkv][kst_tiles][128] fp32 by key tile
  // (tiles numbered per key sequence, rows past a sequence's end hold 0)
  const float* kst_ws;
  int64_t kst_tiles;
};

// Routing bit of key tile j (group j / g); row is a shared- or global-memory
// copy of the query tile's bitmask words, or null (all FP16).
__device__ __forceinline__ bool route8(const uint32_t* row, int g, int j) {
  if (row == nullptr) return false;
  const int G = j / g;
  return (row[G >> 5] >> (G & 31)) & 1u;
}

struct TileInfo {
  int64_t row0;      // first global row of the tile
  int rows;          // valid rows (0: tile absent)
  int nJ;            // key tiles with a visible pair
  int64_t ig;        // global query-tile index
  const uint32_t* mrow;
};

// Row r of an fp16 K or V tile of the INT8 cache, converted in place: the
// slot's upper half holds the int8 code tile as the TMA wrote it (128-byte
// rows, 16-byte chunk c of row r at chunk c ^ (r & 7)); the fp16 tile takes
// the whole slot in the layout the TMA writes for fp16 tiles (two 64-column
// slabs of 128-byte rows, the same chunk swizzle).  Each value is
// fp16_rn(code * scale).  Row r's output in the upper slab covers exactly
// row r's codes, which this thread has read by then, and no other thread
// reads them, so the conversion is race-free in place.  Codes become fp16
// without integer-to-float conversions: XOR 0x80 turns a code x into the
// byte x + 128, which placed under the fp16 exponent byte 0x64 reads as
// 1024 + x + 128 exactly (ulp 1); subtracting 1152 gives x exactly, and one
// fp16 multiply by the fp16 scale rounds the exact product once.
__device__ __forceinline__ void dequant_row_inplace(uint8_t* slot, int r, __half scale, int half_bytes) {
  const int sw = r & 7;
  const __half2 bias = __float2half2_rn(1152.0f);
  const __half2 s2 = __half2half2(scale);
  const uint8_t* codes = slot + half_bytes + r * 128;
  // A rolled loop over the row's eight 16-byte code chunks (small code: this
  // role shares the SM's instruction cache with the softmax and control
  // roles).  Chunk c goes to slab c / 4, chunks 2 (c % 4) and 2 (c % 4) + 1;
  // in slab 1 these overlay code chunks 2 (c - 4) and 2 (c - 4) + 1, which
  // are chunk c itself or ones read in earlier iterations.
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    const uint4 rw = *reinterpret_cast<const uint4*>(codes + ((c ^ sw) << 4));
    const uint32_t w[4] = {rw.x ^ 0x80808080u, rw.y ^ 0x80808080u, rw.z ^ 0x80808080u, rw.w ^ 0x80808080u};
    uint32_t hq[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t lo = __byte_perm(w[q], 0x64646464u, 0x4140u);   // bytes b0, 0x64, b1, 0x64
      uint32_t hi = __byte_perm(w[q], 0x64646464u, 0x4342u);   // bytes b2, 0x64, b3, 0x64
      __half2 vlo = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&lo), bias), s2);
      __half2 vhi = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&hi), bias), s2);
      hq[2 * q] = *reinterpret_cast<uint32_t*>(&vlo);
      hq[2 * q + 1] = *reinterpret_cast<uint32_t*>(&vhi);
    }
    uint8_t* row = slot + (c >> 2) * half_bytes + r * 128;
    const int c0 = 2 * (c & 3);
    *reinterpret_cast<uint4*>(row + ((c0 ^ sw) << 4)) = make_uint4(hq[0], hq[1], hq[2], hq[3]);
    *reinterpret_cast<uint4*>(row + (((c0 + 1) ^ sw) << 4)) = make_uint4(hq[4], hq[5], hq[6], hq[7]);
  }
}

// F8: the 8-bit route is FP8 E4M3 instead of INT8 (a launch with an FP8 bit
// plane and no INT8 plane): the Q8 / K8 maps, tile scales and bitmask are the
// FP8 ones, and the route's QK^T is four kind::f8f6f4 MMAs with an fp32
// result (no seed).  Everything else is the INT8 route's.
template <int D, int EMU, bool DUAL, bool CH, bool CACHE, bool F8 = false, bool TOKS = false>
__global__ void __launch_bounds__(Cfg2<D, CACHE>::THREADS, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ16, const __grid_constant__ CUtensorMap tmQ8,
                     const __grid_constant__ CUtensorMap tmK16, const __grid_constant__ CUtensorMap tmK8,
                     const __grid_constant__ CUtensorMap tmV16, const Params2 p) {
  using C = Cfg2<D, CACHE, TOKS>;
  static_assert(!CACHE || (DUAL && !CH && D == 128), "the INT8 cache runs in the two-issuer mode, d = 128");
  static_assert(!F8 || (!CACHE && !CH && D == 128), "the FP8 route: d = 128, fp16 K / V, routed launches");
  static_assert(!TOKS || (!CACHE && !CH && !F8 && D == 128), "per-token key scales: d = 128, routed launches");
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 8 * C_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 8 * C_COUNT + 4);
  uint32_t* route_words = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + 256);   // [2][MAXW]
  float* ksc = reinterpret_cast<float*>(smem + C::OFF_KSC);                        // [KSC_MAX]
  auto cbar = [&](int i) -> uint32_t { return sbase + C::OFF_CBAR + 8u * static_cast<uint32_t>(i); };
  float* kst = reinterpret_cast<float*>(smem + C::OFF_KST);                        // CACHE: [2][128]
  float* kstt = reinterpret_cast<float*>(smem + C::OFF_KSTT);                      // TOKS: [2][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit (pair P of sequence b, head h).  Grid order: chunk of
  // kv_chunk KV heads (slowest), pair (heaviest first), sequence, query head
  // within the chunk (fastest).  The CTAs resident at any time then read the
  // K / V of one chunk, sized on the host to stay in L2, while the pairs of a
  // chunk still run longest first.
  const int heads_per_chunk = p.kv_chunk * (p.Hq / p.Hkv);
  const int units_per_chunk = heads_per_chunk * p.batch * p.n_pair_max;
  const int chunk = blockIdx.x / units_per_chunk;
  int rest = blockIdx.x - chunk * units_per_chunk;
  const int h = chunk * heads_per_chunk + rest % heads_per_chunk;
  rest /= heads_per_chunk;
  const int b = rest % p.batch;
  const int P = p.n_pair_max - 1 - rest / p.batch;
  const SeqInfo sq = seq_info(p.cu, b, p.Lq, 128);
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
  if (p.cu != nullptr && P == 0 && threadIdx.x == 0 &&
      Lq > static_cast<int64_t>(p.n_qt_max) * 128)
    dev_error(p.err, TM_DEVERR_SEQLEN);
  if (static_cast<int64_t>(2 * P) * 128 >= Lq) return;

  TileInfo ti[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int64_t I = 2 * P + t;
    const int64_t r0 = I * 128;
    ti[t].row0 = sq.start + r0;
    ti[t].rows = r0 < Lq ? static_cast<int>(min(static_cast<int64_t>(128), Lq - r0)) : 0;
    ti[t].ig = sq.tile_base + I;
    ti[t].nJ = 0;
    if (ti[t].rows > 0 && Lk > 0) {
      int64_t jmax = Lk - 1;
      if (p.causal) jmax = min(jmax, r0 + ti[t].rows - 1 + Lk - Lq);
      ti[t].nJ = jmax < 0 ? 0 : static_cast<int>(jmax / BN + 1);
    }
    ti[t].mrow = (p.bitmask && ti[t].rows > 0)
                     ? p.bitmask + static_cast<int64_t>(h) * p.mask_hs + ti[t].ig * p.W : nullptr;
  }
  const int nJ = max(ti[0].nJ, ti[1].nJ);
  const int hk = h / (p.Hq / p.Hkv);
  const int nJA = ti[0].nJ, nJB = ti[1].nJ;
  // Routing words of both query tiles, staged in shared memory when they fit.
  const bool words_in_smem = p.W <= C::MAXW;
  const uint32_t* rrow[2];
#pragma unroll
  for (int t = 0; t < 2; ++t)
    rrow[t] = ti[t].mrow == nullptr ? nullptr : (words_in_smem ? route_words + t * C::MAXW : ti[t].mrow);

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(bar(C_QFULL), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C_SFULL + t), 1);
      mbar_init(bar(C_ODONE + t), 1);
      mbar_init(bar(C_DRAIN + t), 1);
      mbar_init(bar(C_PFULL + t), 4);   // one arrival per softmax warp
    }
    if (CH)
      for (int i = 0; i < 4; ++i) mbar_init(bar(C_SFULL2 + i), 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(bar(C_FULL + s), 1);
      mbar_init(bar(C_EMPTY + s), DUAL ? 2 : 1);
    }
    if (CACHE) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(cbar(CB_KSFULL + s), 128);
        mbar_init(cbar(CB_KSEMPTY + 2 * s), 4);
        mbar_init(cbar(CB_KSEMPTY + 2 * s + 1), 4);
      }
      for (int s = 0; s < C::NSLOT; ++s) mbar_init(cbar(CB_CFULL + s), 1);
    }
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
    if (words_in_smem)
      for (int t = 0; t < 2; ++t)
        if (ti[t].mrow != nullptr)
          for (int w = lane; w < p.W; w += 32) route_words[t * C::MAXW + w] = __ldg(ti[t].mrow + w);
    // the INT8 route's key-tile scales (shared by both query tiles), so that
    // no softmax step waits on a global load for them
    if (!CACHE && !TOKS && (ti[0].mrow != nullptr || ti[1].mrow != nullptr)) {
      const int nst = nJ < C::KSC_MAX ? nJ : C::KSC_MAX;
      for (int j = lane; j < nst; j += 32) ksc[j] = __ldg(p.k_scales + (skq.tile_base + j) * p.Hkv + hk);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // item needs of key tile j (identical in producer and MMA issuer)
  auto needs = [&](int j, bool& r0, bool& r1, bool& n16, bool& n8) {
    const bool a = j < nJA, c = j < nJB;
    r0 = a && route8(rrow[0], p.g, j);
    r1 = c && route8(rrow[1], p.g, j);
    n16 = (a && !r0) || (c && !r1);
    n8 = r0 || r1;
  };

  if (CACHE && warp >= 12) {
    // ======================= dequantisation (CACHE; one key row per thread) ====
    // Walks the ring positions of every key tile in the producer's order
    // ([fp16 K], [int8 K codes], fp16 V): writes the fp16 K tile of a key
    // tile that either query tile routes FP16, and every fp16 V tile, from
    // the cache's codes and per-token scales; the int8 K tiles are the
    // producer's.  Also stages the key tile's per-token K scales for the
    // softmax of INT8 tiles (two stages).  A wait that times out only
    // records the failure: the warps still write and signal every tile, so
    // nothing waits on them forever.
    regs_dec<C::DEQ_REGS>();
    const int r = threadIdx.x - 384;   // key row within the tile
    if (nJ > 0) {
      uint32_t n = 0;
      uint32_t cpar = 0;   // bit s: parity of slot s's next code-barrier phase
      // this row's K and V token scales, loaded one key tile ahead
      auto scales_of = [&](int jj, __half& k_s, __half& v_s) {
        const int64_t kr = static_cast<int64_t>(jj) * BN + r;   // key row within the sequence
        const bool in = jj < nJ && kr < Lk;
        const int64_t tok = kstart + kr;
        k_s = in ? p.k_tok_scale[tok * p.Hkv + hk] : __float2half(0.f);
        v_s = in ? p.v_tok_scale[tok * p.Hkv + hk] : __float2half(0.f);
      };
      __half ksh_next, vsh_next;
      scales_of(0, ksh_next, vsh_next);
      for (int j = 0; j < nJ; ++j) {
        bool r0, r1, n16, n8;
        needs(j, r0, r1, n16, n8);
        const __half ksh = ksh_next, vsh = vsh_next;
        scales_of(j + 1, ksh_next, vsh_next);
        const int s = j & 1;
        if (j >= 2) {   // stage s was key tile j - 2's: both tiles have read it
          if (j - 2 < nJA) mbar_wait_warp(cbar(CB_KSEMPTY + 2 * s), ((j - 2) >> 1) & 1, p.err, abort_flag);
          if (j - 2 < nJB) mbar_wait_warp(cbar(CB_KSEMPTY + 2 * s + 1), ((j - 2) >> 1) & 1, p.err, abort_flag);
        }
        kst[s * 128 + r] = __half2float(ksh);
        mbar_arrive(cbar(CB_KSFULL + s));
        // An fp16 tile: wait for its code tile, convert it in place (rows
        // past the key sequence get scale 0, so they read as zeros), then
        // hand the slot to the MMA side.  The slot itself was acquired by
        // the producer (its release barrier), which the code barrier orders.
        auto convert = [&](__half scale) {
          const uint32_t slot = n % C::NSLOT;
          ++n;
          mbar_wait_warp(cbar(CB_CFULL + slot), (cpar >> slot) & 1u, p.err, abort_flag);
          cpar ^= 1u << slot;
          dequant_row_inplace(smem + C::OFF_SLOT + slot * C::SLOT, r, scale, C::HALF);
          fence_async_shared();   // generic-proxy stores, read by tcgen05.mma
          named_bar_sync(NB_DEQ, 128);
          if (r == 0) mbar_arrive(bar(C_FULL + slot));
        };
        if (n16) convert(ksh);
        if (n8) ++n;   // the producer's int8 K tile
        convert(vsh);
      }
    }
  } else if (warp >= 8) {
   regs_dec<C::CONTROL_REGS>();
   if (warp == 8) {
    // ======================= TMA producer =======================
    if (lane == 0 && nJ > 0) {
#ifndef TM_TRACE_HELPER
      TM_TRACE_DECL
      TM_TRACE_EV(2, EV_START);
#endif
      bool any8[2] = {false, false};
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (ti[t].mrow != nullptr)
          for (int w = 0; w < p.W; ++w) any8[t] |= (__ldg(ti[t].mrow + w) != 0u);
      uint32_t qbytes = 0;
#pragma unroll
      for (int t = 0; t < 2; ++t) qbytes += (ti[t].rows > 0 ? C::Q16_BYTES : 0) + (any8[t] ? C::Q8_BYTES : 0);
      // Q is read once (evict first); K / V are re-read by every query tile
      // of the KV head (evict last).
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_arrive_expect_tx(bar(C_QFULL), qbytes);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (ti[t].rows == 0) continue;
        const int32_t qr = static_cast<int32_t>(ti[t].row0);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d_hint(sbase + C::OFF_Q16 + t * C::Q16_BYTES + hh * C::HALF, &tmQ16, bar(C_QFULL), hh * 64, h,
                           qr, pol_q);
        if (any8[t]) tma_load_3d_hint(sbase + C::OFF_Q8 + t * C::Q8_BYTES, &tmQ8, bar(C_QFULL), 0, h, qr, pol_q);
      }

      uint32_t n = 0;   // ring position
      auto acquire = [&](uint32_t& slot) -> bool {
        slot = n % C::NSLOT;
        const uint32_t lap = n / C::NSLOT;
        if (lap > 0 && !mbar_wait(bar(C_EMPTY + slot), (lap - 1) & 1, p.err, abort_flag)) return false;
        ++n;
#ifndef TM_TRACE_HELPER
        TM_TRACE_EV(2, EV_ACQUIRED);
#endif
        return true;
      };
      bool ok = true;
      for (int j = 0; ok && j < nJ; ++j) {
        bool r0, r1, n16, n8;
        needs(j, r0, r1, n16, n8);
        const int32_t krow = static_cast<int32_t>(kstart + static_cast<int64_t>(j) * BN);
        uint32_t s;
        if (CACHE) {
          // Ring positions of this key tile: [fp16 K], [int8 K codes], fp16 V.
          // For an fp16 tile the producer brings the int8 code tile into the
          // upper half of the slot (signalled on the slot's code barrier);
          // the dequantisation warps turn it into the fp16 tile in place and
          // signal the slot's full barrier.  An int8 K tile lands at the
          // slot's start as usual.  (tmV16 holds the V codes' map here.)
          if (n16) {
            if (!(ok = acquire(s))) break;
            mbar_arrive_expect_tx(cbar(CB_CFULL + s), BN * D);
            tma_load_3d_hint(sbase + C::OFF_SLOT + s * C::SLOT + C::SLOT / 2, &tmK8, cbar(CB_CFULL + s), 0, hk,
                             krow, pol_kv);
          }
          if (n8) {
            if (!(ok = acquire(s))) break;
            mbar_arrive_expect_tx(bar(C_FULL + s), BN * D);
            tma_load_3d_hint(sbase + C::OFF_SLOT + s * C::SLOT, &tmK8, bar(C_FULL + s), 0, hk, krow, pol_kv);
          }
          if (!(ok = acquire(s))) break;
          mbar_arrive_expect_tx(cbar(CB_CFULL + s), BN * D);
          tma_load_3d_hint(sbase + C::OFF_SLOT + s * C::SLOT + C::SLOT / 2, &tmV16, cbar(CB_CFULL + s), 0, hk, krow,
                           pol_kv);
          continue;
        }
        if (n16) {
          if (!(ok = acquire(s))) break;
          mbar_arrive_expect_tx(bar(C_FULL + s), C::SLOT);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d_hint(sbase + C::OFF_SLOT + s * C::SLOT + hh * C::HALF, &tmK16, bar(C_FULL + s), hh * 64, hk,
                             krow, pol_kv);
        }
        if (n8) {
          if (!(ok = acquire(s))) break;
          mbar_arrive_expect_tx(bar(C_FULL + s), BN * D);
          tma_load_3d_hint(sbase + C::OFF_SLOT + s * C::SLOT, &tmK8, bar(C_FULL + s), 0, hk, krow, pol_kv);
        }
        if (!(ok = acquire(s))) break;
        mbar_arrive_expect_tx(bar(C_FULL + s), C::SLOT);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d_hint(sbase + C::OFF_SLOT + s * C::SLOT + hh * C::HALF, &tmV16, bar(C_FULL + s), hh * 64, hk,
                           krow, pol_kv);
      }
      // Drain: every issued copy has landed before the CTA may exit.
      volatile int never = 0;
      mbar_wait(bar(C_QFULL), 0, p.err, &never);
      for (uint32_t i = (n > C::NSLOT ? n - C::NSLOT : 0); i < n; ++i)
        mbar_wait(bar(C_FULL + i % C::NSLOT), (i / C::NSLOT) & 1, p.err, &never);
    }
   } else if (DUAL) {
   if (warp == 9 || warp == 10) {
    // ======================= tcgen05 issuers (warp 9: tile A, warp 10: tile B) ====
    // One issuing warp per query tile, so that neither tile's P.V and next
    // S wait behind the other tile's MMAs.  An issuing warp never touches
    // shared memory inside its loop: on this SM a barrier poll (or any
    // shared-memory access) by the thread that issues tcgen05.mma holds back
    // its next MMA by ~200 cycles while the MMAs saturate the shared-memory
    // port, and the MMA queue is too short to cover that.  It learns that P
    // is stored from its softmax warpgroup at named barrier NB_P + t, and
    // that K / V landed from the wait helper at NB_KV + t.  One elected lane
    // issues each group of MMAs and its commits.  Each ring slot is released
    // by two commits (one per query tile); a tile past its last key tile
    // leaves its share to the other tile's issuer.
    const int t = warp - 9;
    const int nJt = t == 0 ? nJA : nJB;
    const int nJo = t == 0 ? nJB : nJA;
    if (nJt > 0) {
      TM_TRACE_DECL
      const bool tracer = lane == 0 && t == 0;
      if (tracer) TM_TRACE_EV(3, EV_START);
      auto kv_handoff = [&]() { named_bar_sync(NB_KV + t, 64); };
      auto p_handoff = [&]() { named_bar_sync(NB_P + t, 160); };
      kv_handoff();   // Q tiles landed
      uint32_t n = 0;
      auto take = [&](uint32_t& slot) {
        slot = n % C::NSLOT;
        ++n;
      };
      int wwin = -1;
      uint32_t rw0 = 0, rw1 = 0;
      auto route_reg = [&](int j, bool& r0, bool& r1, bool& n16, bool& n8) {
        const bool a = j < nJA, c = j < nJB;
        const int G = j / p.g;
        if ((G >> 5) != wwin) {   // one shared-memory read per 32 routing groups
          wwin = G >> 5;
          rw0 = rrow[0] != nullptr ? rrow[0][wwin] : 0u;
          rw1 = rrow[1] != nullptr ? rrow[1][wwin] : 0u;
        }
        r0 = a && ((rw0 >> (G & 31)) & 1u);
        r1 = c && ((rw1 >> (G & 31)) & 1u);
        n16 = (a && !r0) || (c && !r1);
        n8 = r0 || r1;
      };
      // release a ring slot: this tile's share, plus the other tile's when
      // that tile has no key tile jj
      auto release = [&](uint32_t slot, int jj) {
        if (elect_one()) {
          tc_commit(bar(C_EMPTY + slot));
          if (jj >= nJo) tc_commit(bar(C_EMPTY + slot));
        }
        __syncwarp();
      };
      const uint32_t d_s = tmem + C::s_col(t), d_o = tmem + C::o_col(t);
      const uint64_t sd[3] = {seed_desc(sbase + C::OFF_SEED), seed_desc(sbase + C::OFF_SEED + 128),
                              seed_desc(sbase + C::OFF_SEED + 256)};
      auto issue_s = [&](bool i8, uint32_t kslot) {
        const uint32_t kb = sbase + C::OFF_SLOT + kslot * C::SLOT;
        if (i8) {
          const uint32_t qa = sbase + C::OFF_Q8 + t * C::Q8_BYTES;
          uint64_t ad[D / 32], bd[D / 32];
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            ad[kk] = smem_desc(qa + kk * 32, 16, C::SBO8, C::SW8);
            bd[kk] = smem_desc(kb + kk * 32, 16, C::SBO8, C::SW8);
          }
          if (elect_one()) {
            if constexpr (F8) mma_f8_ss_n<D / 32>(d_s, ad, bd, C::IDESC_F8, 0u);
            else mma_i8_exact_n<D / 32>(d_s, sd, C::IDESC_S16, ad, bd, C::IDESC_S8);
            tc_commit(bar(C_SFULL + t));
          }
        } else {
          const uint32_t qa = sbase + C::OFF_Q16 + t * C::Q16_BYTES;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::HALF + (kk & 3) * 32;
              mma_f16_ss(d_s, smem_desc(qa + off, 16, 1024, kSwizzle128),
                         smem_desc(kb + off, 16, 1024, kSwizzle128), C::IDESC_S16, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar(C_SFULL + t));
          }
        }
        __syncwarp();
      };
      auto issue_pv = [&](int jj, uint32_t vslot) {
        p_handoff();        // softmax t stored P_t(jj)
        if (tracer) TM_TRACE_EV(3, EV_P_SEEN);
        tc_fence_after();   // orders the softmax warps' TMEM stores of P before the MMA reads it
        const uint32_t vb = sbase + C::OFF_SLOT + vslot * C::SLOT;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_f16_ts(d_o, d_s + kk * 8, smem_desc(vb + kk * 2048, C::HALF, 1024, kSwizzle128), C::IDESC_PV,
                       (jj > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(C_ODONE + t));
        }
        __syncwarp();
        release(vslot, jj);
      };
      if constexpr (CH) {
        // Chunked mode: each 128-key tile is two 64-key chunks, c = 2J and
        // 2J + 1, whose scores alternate between the two 64-column halves
        // ("slots") of this tile's score columns; P(c) overwrites its slot,
        // and S(c + 2) is issued right behind P.V(c) into the same slot.
        auto issue_s_ch = [&](bool i8, uint32_t kslot, int c) {
          const uint32_t kb = sbase + C::OFF_SLOT + kslot * C::SLOT + (c & 1) * 8192;   // key rows 64 (c & 1) ..
          const uint32_t d_c = d_s + 64u * static_cast<uint32_t>(c & 1);
          if (i8) {
            const uint32_t qa = sbase + C::OFF_Q8 + t * C::Q8_BYTES;
            uint64_t ad[D / 32], bd[D / 32];
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
              ad[kk] = smem_desc(qa + kk * 32, 16, C::SBO8, C::SW8);
              bd[kk] = smem_desc(kb + kk * 32, 16, C::SBO8, C::SW8);
            }
            if (elect_one()) {
              mma_i8_exact_n<D / 32>(d_c, sd, C::IDESC_S16_64, ad, bd, C::IDESC_S8_64);
              tc_commit(bar(C_SFULL2 + 2 * t + (c & 1)));
            }
          } else {
            const uint32_t qa = sbase + C::OFF_Q16 + t * C::Q16_BYTES;
            uint64_t ad[D / 16], bd[D / 16];
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::HALF + (kk & 3) * 32;
              ad[kk] = smem_desc(qa + off, 16, 1024, kSwizzle128);
              bd[kk] = smem_desc(kb + off, 16, 1024, kSwizzle128);
            }
            if (elect_one()) {
              mma_f16_ss_n<D / 16>(d_c, ad, bd, C::IDESC_S16_64, 0u);
              tc_commit(bar(C_SFULL2 + 2 * t + (c & 1)));
            }
          }
          __syncwarp();
        };
        auto issue_pv_ch = [&](int c, uint32_t vslot) {
          const uint32_t vb = sbase + C::OFF_SLOT + vslot * C::SLOT;
          uint32_t at[4];
          uint64_t bd[4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            at[kk] = d_s + 64u * static_cast<uint32_t>(c & 1) + kk * 8;
            bd[kk] = smem_desc(vb + ((c & 1) * 4 + kk) * 2048, C::HALF, 1024, kSwizzle128);
          }
          p_handoff();        // softmax t stored P_t(c)
          if (tracer) TM_TRACE_EV(3, EV_P_SEEN);
          tc_fence_after();   // orders the softmax warps' TMEM stores of P before the MMA reads it
          if (elect_one()) {
            mma_f16_ts_n<4>(d_o, at, bd, C::IDESC_PV, c > 0 ? 1u : 0u);
            tc_commit(bar(C_ODONE + t));
          }
          __syncwarp();
        };
        uint32_t v_prev = 0;
        for (int j = 0; j < nJt; ++j) {
          bool r0, r1, n16, n8;
          route_reg(j, r0, r1, n16, n8);
          uint32_t s16 = 0, s8 = 0, sv = 0;
          if (n16) take(s16);
          if (n8) take(s8);
          take(sv);
          kv_handoff();   // K tiles of j (and V of j-1) landed
          const bool r = t == 0 ? r0 : r1;
          const uint32_t ks = r ? s8 : s16;
          if (j > 0) issue_pv_ch(2 * j - 2, v_prev);
          if (tracer) TM_TRACE_EV(3, EV_K_READY);
          if (t == 1 && j == 0 && nJA > 0) named_bar_sync(NB_START, 160);
          issue_s_ch(r, ks, 2 * j);
          if (j > 0) {
            issue_pv_ch(2 * j - 1, v_prev);
            release(v_prev, j - 1);
          }
          issue_s_ch(r, ks, 2 * j + 1);
          if (tracer) TM_TRACE_EV(3, EV_S_A);
          if (n16) release(s16, j);
          if (n8) release(s8, j);
          v_prev = sv;
        }
        kv_handoff();   // V of the last key tile landed
        issue_pv_ch(2 * nJt - 2, v_prev);
        issue_pv_ch(2 * nJt - 1, v_prev);
        release(v_prev, nJt - 1);
      } else {
        uint32_t v_prev = 0;
        for (int j = 0; j < nJt; ++j) {
          bool r0, r1, n16, n8;
          route_reg(j, r0, r1, n16, n8);
          uint32_t s16 = 0, s8 = 0, sv = 0;
          if (n16) take(s16);
          if (n8) take(s8);
          take(sv);
          kv_handoff();   // K tiles of j (and V of j-1) landed
          if (CACHE) tc_fence_after();   // tiles the dequantisation warps wrote
          // P.V of the previous key tile first (S_t(j) overwrites P_t(j-1))
          if (j > 0) issue_pv(j - 1, v_prev);
          if (tracer) TM_TRACE_EV(3, EV_K_READY);
          const bool r = t == 0 ? r0 : r1;
          // Tile B starts half a period behind tile A: its first S waits until
          // softmax A has stored P_A(0), so that the two tiles' softmax and
          // MMA phases alternate instead of running in lockstep.  (This waits
          // only on S_A(0); nothing it waits for depends on tile B.)
          if (t == 1 && j == 0 && nJA > 0) named_bar_sync(NB_START, 160);
          issue_s(r, r ? s8 : s16);
          if (tracer) TM_TRACE_EV(3, EV_S_A);
          if (n16) release(s16, j);
          if (n8) release(s8, j);
          v_prev = sv;
        }
        kv_handoff();   // V of the last key tile landed
        if (CACHE) tc_fence_after();
        issue_pv(nJt - 1, v_prev);
      }
      if (elect_one()) tc_commit(bar(C_DRAIN + t));
      __syncwarp();
      if (lane == 0) {
        volatile int never = 0;
        mbar_wait(bar(C_DRAIN + t), 0, p.err, &never);
      }
      __syncwarp();
    }
  } else if (warp == 11) {
    // ======================= wait helper =======================
    // Makes both issuers' operand waits (Q, then per key tile j: K of j and
    // V of j-1, then the last V) and meets issuer t at named barrier
    // NB_KV + t after each, tile A's handoff of a round before tile B's.  A
    // wait that times out or sees the abort flag only records the failure:
    // the helper still takes every handoff, so no warp is left at a barrier,
    // and the remaining MMAs run on stale operands of a launch that reports
    // the error.
    if (nJ > 0) {
#ifdef TM_TRACE_HELPER
      TM_TRACE_DECL
#endif
      auto wait1 = [&](uint32_t b, uint32_t par) {
#ifdef TM_TRACE_HELPER
        if (lane == 0) TM_TRACE_EV(2, EV_HW_KV_BEGIN);
#endif
        if (lane == 0) mbar_wait(b, par, p.err, abort_flag);
#ifdef TM_TRACE_HELPER
        if (lane == 0) TM_TRACE_EV(2, EV_HW_KV_END);
#endif
      };
      auto handoff = [&](int t) {
        __syncwarp();
        named_bar_sync(NB_KV + t, 64);
      };
      wait1(bar(C_QFULL), 0);
      if (nJA > 0) handoff(0);
      if (nJB > 0) handoff(1);
      uint32_t n = 0;
      auto take = [&](uint32_t& slot, uint32_t& par) {
        slot = n % C::NSLOT;
        par = (n / C::NSLOT) & 1;
        ++n;
      };
      uint32_t sv_prev = 0, pv_prev = 0;
      for (int j = 0; j < nJ; ++j) {
        bool r0, r1, n16, n8;
        needs(j, r0, r1, n16, n8);
        uint32_t s16 = 0, s8 = 0, sv = 0, par16 = 0, par8 = 0, parv = 0;
        if (n16) take(s16, par16);
        if (n8) take(s8, par8);
        take(sv, parv);
        if (j > 0) wait1(bar(C_FULL + sv_prev), pv_prev);
        if (n16) wait1(bar(C_FULL + s16), par16);
        if (n8) wait1(bar(C_FULL + s8), par8);
        if (j < nJA) handoff(0);
        if (j < nJB) handoff(1);
        // after a tile's last key tile: the V of that key tile
        if (j == nJA - 1 || j == nJB - 1) wait1(bar(C_FULL + sv), parv);
        if (j == nJA - 1) handoff(0);
        if (j == nJB - 1) handoff(1);
        sv_prev = sv;
        pv_prev = parv;
      }
    }
   }
   } else {
   if (warp == 9) {
    // ======================= tcgen05 issuer =======================
    // The issuing warp never touches shared memory inside its loop: on this
    // SM a barrier poll (or any shared-memory access) by the thread that
    // issues tcgen05.mma holds back its next MMA for ~200 cycles while the
    // MMAs saturate the shared-memory port, and the MMA queue is too short to
    // cover that.  Every mbarrier wait is made by the wait helper (warp 10),
    // which then meets this warp at named barrier 1; the two walk the same
    // sequence of handoffs.  Routing words are kept in registers.  One
    // elected lane issues each group of MMAs and its commits.
    if (nJ > 0) {
      TM_TRACE_DECL
      const bool tracer = lane == 0;
      if (tracer) TM_TRACE_EV(3, EV_START);
      auto handoff = [&]() { named_bar_sync(1, 64); };
      handoff();   // Q tiles landed
      uint32_t n = 0;
      auto take = [&](uint32_t& slot) {
        slot = n % C::NSLOT;
        ++n;
      };
      int wwin = -1;
      uint32_t rw0 = 0, rw1 = 0;
      auto route_reg = [&](int j, bool& r0, bool& r1, bool& n16, bool& n8) {
        const bool a = j < nJA, c = j < nJB;
        const int G = j / p.g;
        if ((G >> 5) != wwin) {   // one shared-memory read per 32 routing groups
          wwin = G >> 5;
          rw0 = rrow[0] != nullptr ? rrow[0][wwin] : 0u;
          rw1 = rrow[1] != nullptr ? rrow[1][wwin] : 0u;
        }
        r0 = a && ((rw0 >> (G & 31)) & 1u);
        r1 = c && ((rw1 >> (G & 31)) & 1u);
        n16 = (a && !r0) || (c && !r1);
        n8 = r0 || r1;
      };
      const uint64_t sd[3] = {seed_desc(sbase + C::OFF_SEED), seed_desc(sbase + C::OFF_SEED + 128),
                              seed_desc(sbase + C::OFF_SEED + 256)};
      auto issue_s = [&](int t, bool i8, uint32_t kslot) {
        const uint32_t d_tmem = tmem + C::s_col(t);
        const uint32_t kb = sbase + C::OFF_SLOT + kslot * C::SLOT;
        if (i8) {
          const uint32_t qa = sbase + C::OFF_Q8 + t * C::Q8_BYTES;
          uint64_t ad[D / 32], bd[D / 32];
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            ad[kk] = smem_desc(qa + kk * 32, 16, C::SBO8, C::SW8);
            bd[kk] = smem_desc(kb + kk * 32, 16, C::SBO8, C::SW8);
          }
          if (elect_one()) {
            if constexpr (F8) mma_f8_ss_n<D / 32>(d_tmem, ad, bd, C::IDESC_F8, 0u);
            else mma_i8_exact_n<D / 32>(d_tmem, sd, C::IDESC_S16, ad, bd, C::IDESC_S8);
            tc_commit(bar(C_SFULL + t));
          }
        } else {
          const uint32_t qa = sbase + C::OFF_Q16 + t * C::Q16_BYTES;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::HALF + (kk & 3) * 32;
              mma_f16_ss(d_tmem, smem_desc(qa + off, 16, 1024, kSwizzle128),
                         smem_desc(kb + off, 16, 1024, kSwizzle128), C::IDESC_S16, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar(C_SFULL + t));
          }
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int jj, uint32_t vslot) {
        handoff();          // softmax t released P_t(jj)
        if (tracer) TM_TRACE_EV(3, EV_P_SEEN);
        tc_fence_after();   // orders the softmax warps' TMEM stores of P before the MMA reads it
        const uint32_t vb = sbase + C::OFF_SLOT + vslot * C::SLOT;
        const uint32_t a_tmem = tmem + C::s_col(t);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            mma_f16_ts(tmem + C::o_col(t), a_tmem + kk * 8, smem_desc(vb + kk * 2048, C::HALF, 1024, kSwizzle128),
                       C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
#ifdef TM_TRACE_MMA
            TM_TRACE_EV(3, EV_MMA_ISSUED);
#endif
          }
          tc_commit(bar(C_ODONE + t));
        }
        __syncwarp();
      };
      auto commit1 = [&](uint32_t b) {
        if (elect_one()) tc_commit(b);
        __syncwarp();
      };
      uint32_t v_prev = 0;
      for (int j = 0; j < nJ; ++j) {
        bool r0, r1, n16, n8;
        route_reg(j, r0, r1, n16, n8);
        // P.V of tile A for the previous key tile first: its operands (P_A,
        // V) are ready as soon as softmax A releases P, and the wait for this
        // key tile's K then overlaps its execution.
        if (j > 0 && j - 1 < nJA) issue_pv(0, j - 1, v_prev);
        if (tracer) TM_TRACE_EV(3, EV_PV_A);
        uint32_t s16 = 0, s8 = 0, sv = 0;
        if (n16) take(s16);
        if (n8) take(s8);
        take(sv);
        handoff();   // K tiles of j landed
        if (tracer) TM_TRACE_EV(3, EV_K_READY);
        if (j < nJA) issue_s(0, r0, r0 ? s8 : s16);
        if (tracer) TM_TRACE_EV(3, EV_S_A);
        if (j > 0 && j - 1 < nJB) issue_pv(1, j - 1, v_prev);
        if (tracer) TM_TRACE_EV(3, EV_PV_B);
        if (j > 0) commit1(bar(C_EMPTY + v_prev));
        if (j < nJB) issue_s(1, r1, r1 ? s8 : s16);
        if (tracer) TM_TRACE_EV(3, EV_S_B);
        if (n16) commit1(bar(C_EMPTY + s16));
        if (n8) commit1(bar(C_EMPTY + s8));
        handoff();   // V of j landed (its P.V is issued next round)
        if (tracer) TM_TRACE_EV(3, EV_V_READY);
        v_prev = sv;
      }
      if (nJ - 1 < nJA) issue_pv(0, nJ - 1, v_prev);
      if (nJ - 1 < nJB) issue_pv(1, nJ - 1, v_prev);
      commit1(bar(C_EMPTY + v_prev));
      commit1(bar(C_DRAIN));
      if (lane == 0) {
        volatile int never = 0;
        mbar_wait(bar(C_DRAIN), 0, p.err, &never);
      }
      __syncwarp();
    }
  } else if (warp == 10) {
    // ======================= wait helper =======================
    // Makes the issuer's mbarrier waits (operands landed, P released) in the
    // issuer's order and meets it at named barrier 1 after each.  A wait that
    // times out or sees the abort flag only records the failure: the helper
    // still takes every handoff, so neither warp is left at the barrier, and
    // the issuer's remaining MMAs run on stale operands whose results the
    // failed launch discards.
    if (nJ > 0) {
      auto wait1 = [&](uint32_t b, uint32_t par) {
        if (lane == 0) mbar_wait(b, par, p.err, abort_flag);
      };
      auto handoff = [&]() {
        __syncwarp();
        named_bar_sync(1, 64);
      };
      auto wait_p = [&](int t, int jj) {   // P_t(jj) released
        wait1(bar(C_PFULL + t), jj & 1);
        handoff();
      };
      wait1(bar(C_QFULL), 0);
      handoff();
      uint32_t n = 0;
      auto take = [&](uint32_t& slot, uint32_t& par) {
        slot = n % C::NSLOT;
        par = (n / C::NSLOT) & 1;
        ++n;
      };
      for (int j = 0; j < nJ; ++j) {
        bool r0, r1, n16, n8;
        needs(j, r0, r1, n16, n8);
        if (j > 0 && j - 1 < nJA) wait_p(0, j - 1);
        uint32_t s16 = 0, s8 = 0, sv = 0, par16 = 0, par8 = 0, parv = 0;
        if (n16) take(s16, par16);
        if (n8) take(s8, par8);
        take(sv, parv);
        if (n16) wait1(bar(C_FULL + s16), par16);
        if (n8) wait1(bar(C_FULL + s8), par8);
        handoff();
        if (j > 0 && j - 1 < nJB) wait_p(1, j - 1);
        wait1(bar(C_FULL + sv), parv);
        handoff();
      }
      if (nJ - 1 < nJA) wait_p(0, nJ - 1);
      if (nJ - 1 < nJB) wait_p(1, nJ - 1);
    }
   }
   }
  } else {
    // ======================= softmax (warpgroup t = tile t) =======================
    regs_inc<C::SOFTMAX_REGS>();
    const int t = warp >> 2;
    const TileInfo& T = ti[t];
    const int r = threadIdx.x & 127;                 // row in the tile = TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_addr + C::s_col(t);
    const uint32_t o_addr = lane_addr + C::o_col(t);
    const bool row_ok = r < T.rows;
    const int64_t i_row = static_cast<int64_t>(2 * P + t) * 128 + r;
    int64_t lim = -1;
    if (row_ok) lim = p.causal ? min(Lk - 1, i_row + Lk - Lq) : Lk - 1;
    float c8_row = 0.f;
    if (T.mrow != nullptr) c8_row = __ldg(p.q_scales + T.ig * p.Hq + h) * p.scale_log2;
    const SeqInfo sk = seq_info(p.cu_k, b, p.Lk, BN);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // TOKS: this warpgroup's row of key scales and the next key tile's scale
    // of column r (loaded one key tile ahead)
    float* kst_row = kstt + 128 * t;
    const float* kst_src = TOKS ? p.kst_ws + (static_cast<int64_t>(hk) * p.kst_tiles + sk.tile_base) * 128 + r
                                : nullptr;
    float kst_next = 0.f;
    if (TOKS) {
      if (T.nJ > 0) kst_row[r] = __ldg(kst_src);
      if (T.nJ > 1) kst_next = __ldg(kst_src + 128);
    }
    TM_TRACE_DECL
#ifndef TM_TRACE_WARP
#define TM_TRACE_WARP 0
#endif
    const bool tracer = (threadIdx.x & 127) == 32 * TM_TRACE_WARP;
    TM_SM_EV(EV_START);
    TM_PH_DECL
    if constexpr (CH) {
      // Chunked mode: 64-key chunks c = 0 .. 2 nJ - 1 alternating between
      // the two 64-column slots of this tile's score columns.
      constexpr int HN = 64;
      for (int c = 0; c < 2 * T.nJ; ++c) {
        const int j = c >> 1, sl = c & 1;
        const uint32_t s_c = s_addr + HN * sl;
        const bool i8 = route8(rrow[t], p.g, j);
        float cs = p.scale_log2;
        if (i8) {
          const float ks = j < C::KSC_MAX ? ksc[j] : __ldg(p.k_scales + (sk.tile_base + j) * p.Hkv + hk);
          cs = fmaxf(c8_row * ks, 1e-30f);
        }
        // No early exit: the issuer expects one P handoff per chunk.
        if (!mbar_wait(bar(C_SFULL2 + 2 * t + sl), (c >> 1) & 1, p.err, abort_flag)) ok = false;
        tc_fence_after();
        TM_PH(0);
        TM_SM_EV(EV_S_READY);
        __syncwarp();
        float x[HN];
        {
          uint32_t u[HN];
#pragma unroll
          for (int cc = 0; cc < HN / 32; ++cc) tmem_ld32p(s_c + cc * 32, u + cc * 32);
          tmem_wait_ld_regs<HN>(u);
          TM_PH(1);
          // INT8 scores arrive in fp32 like FP16 ones (see mma_i8_exact_n)
#pragma unroll
          for (int e = 0; e < HN; ++e) x[e] = __uint_as_float(u[e]);
        }
        const int64_t nv64 = lim - static_cast<int64_t>(c) * HN + 1;
        const int nv = nv64 <= 0 ? 0 : (nv64 >= HN ? HN : static_cast<int>(nv64));
        if (!__all_sync(0xffffffffu, nv == HN)) {
#pragma unroll
          for (int e = 0; e < HN; ++e) x[e] = (e < nv) ? x[e] : -INFINITY;
        }
        float alpha = 1.f;
        if (nv > 0) {
          const float mt = row_max<HN>(x) * cs;
          if (mt > m_used + kLazyRescaleLog2) {
            alpha = ex2_approx(m_used - mt);
            m_used = mt;
          }
        }
        const float msub = (m_used == -INFINITY) ? 0.f : m_used;
        TM_PH(2);
        const uint64_t c2 = f2pack(cs, cs);
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
        }
        {
          const uint64_t s2 = f2add(f2add(acc2[0], acc2[1]), f2add(acc2[2], acc2[3]));
          float s0, s1;
          f2unpack(s2, s0, s1);
          l = l * alpha + (s0 + s1);
        }
        TM_PH(3);
        __syncwarp();
        tmem_st32p(s_c, pk);   // P_t(c) over the first 32 columns of its slot
        // O is rescaled only when a row of this warp raised its running max.
        // Then P.V(c-1) must have completed: S(c) was issued after P.V(c-2)
        // and has completed, so phases <= c-2 of the P.V barrier are done
        // and waiting for phase c-1 by parity is unambiguous.
        if (c > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!mbar_wait(bar(C_ODONE + t), (c - 1) & 1, p.err, abort_flag)) ok = false;
          tc_fence_after();
          __syncwarp();
          uint32_t o[D];
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_ld32p(o_addr + cc * 32, o + cc * 32);
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
          for (int cc = 0; cc < D / 32; ++cc) tmem_st32p(o_addr + cc * 32, o + cc * 32);
        }
        tmem_wait_st();
        tc_fence_before();
        TM_PH(4);
        __syncwarp();
        // Tile B's first S waits for P_A(0) (NB_START).  Signal it before the
        // handoff below: issuer A takes P_A(0) only after K of key tile 1 has
        // landed, which can need the ring slot that tile B releases after its
        // first S.
        if (t == 0 && c == 0 && ti[1].nJ > 0) named_bar_arrive(NB_START, 160);
        // P_t(c) stored: meet issuer t.  Both sides wait, so the softmax can
        // never signal chunk c+1 before the issuer has taken chunk c (its S
        // is computed one chunk ahead).
        named_bar_sync(NB_P + t, 160);
        TM_PH(5);
        TM_SM_EV(EV_P_RELEASED);
      }
    } else {
    for (int j = 0; j < T.nJ; ++j) {
      const bool i8 = route8(rrow[t], p.g, j);
      float c = p.scale_log2;
      if (i8) {
        if (CACHE || TOKS) {
          c = fmaxf(c8_row, 1e-30f);   // the per-token key scales multiply the scores per column below
        } else {
          const float ks = j < C::KSC_MAX ? ksc[j] : __ldg(p.k_scales + (sk.tile_base + j) * p.Hkv + hk);
          c = fmaxf(c8_row * ks, 1e-30f);
        }
      }
      // No early exit: the issuer expects one P handoff per key tile, so a
      // failed wait only marks the launch failed and the loop runs on.
      if (!mbar_wait(bar(C_SFULL + t), j & 1, p.err, abort_flag)) ok = false;
      tc_fence_after();
      TM_PH(0);
      TM_SM_EV(EV_S_READY);
      __syncwarp();
      float x[BN];
      {
        uint32_t u[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32p(s_addr + cc * 32, u + cc * 32);
        tmem_wait_ld_regs<BN>(u);
        TM_PH(1);
        TM_SM_EV(EV_SLOADED);
        // Never taken (sched_zero is 0 in every launch).  The branch only
        // changes how the compiler schedules this step: without it the same
        // launches measured 5-7 % slower (routing sweep, every INT8 share).
        if (p.sched_zero != 0) {
#pragma unroll
          for (int e = 0; e < BN; ++e) u[e] += static_cast<uint32_t>(p.sched_zero);
        }
        // INT8 scores arrive in fp32 like FP16 ones (see mma_i8_exact_n)
#pragma unroll
        for (int e = 0; e < BN; ++e) x[e] = __uint_as_float(u[e]);
      }
      if constexpr (CACHE) {
        // INT8 cache: the score of key column e is acc * s_k[e] * s_q * sigma;
        // s_k of this key tile's tokens is staged in stage j & 1
        const int ks_stage = j & 1;
        // Every key tile waits for its stage, FP16 ones too: a warp must not
        // release stage j & 1 for key tile j before the dequantisation warps
        // have written it, or that barrier would run two phases ahead of
        // their wait for key tile j - 2.
        if (!mbar_wait(cbar(CB_KSFULL + ks_stage), (j >> 1) & 1, p.err, abort_flag)) ok = false;
        if (i8) {
          const float2* ks2 = reinterpret_cast<const float2*>(kst + ks_stage * 128);
#pragma unroll
          for (int e = 0; e < BN; e += 2) {
            const float2 kk = ks2[e >> 1];
            f2unpack(f2mul(f2pack(x[e], x[e + 1]), f2pack(kk.x, kk.y)), x[e], x[e + 1]);
            // eight scale pairs in flight at most (keeps them out of the
            // registers the scores need)
            if ((e & 15) == 14) asm volatile("" ::: "memory");
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cbar(CB_KSEMPTY + 2 * ks_stage + t));   // this warp is done with the stage
      }
      if constexpr (TOKS) {
        // Per-token K scales of key tile j, in this warpgroup's row: thread r
        // wrote scale r during the previous key tile (or before the loop);
        // the first barrier makes the row visible, the second lets thread r
        // overwrite its entry with key tile j + 1's scale once every thread
        // has read the row.  Both run for every key tile, FP16 ones too.
        named_bar_sync(NB_KST + t, 128);
        if (i8) {
          const float4* kp = reinterpret_cast<const float4*>(kst_row);
#pragma unroll
          for (int e = 0; e < BN; e += 4) {
            const float4 kk = kp[e >> 2];
            f2unpack(f2mul(f2pack(x[e], x[e + 1]), f2pack(kk.x, kk.y)), x[e], x[e + 1]);
            f2unpack(f2mul(f2pack(x[e + 2], x[e + 3]), f2pack(kk.z, kk.w)), x[e + 2], x[e + 3]);
          }
        }
        named_bar_sync(NB_KST + t, 128);
        kst_row[r] = kst_next;
        kst_next = (j + 2 < T.nJ) ? __ldg(kst_src + (j + 2) * 128) : 0.f;
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
        if (mt > m_used + kLazyRescaleLog2) {
          alpha = ex2_approx(m_used - mt);
          m_used = mt;
        }
      }
      const float msub = (m_used == -INFINITY) ? 0.f : m_used;
      TM_PH(2);
      TM_SM_EV(EV_MAXED);
      const uint64_t c2 = f2pack(c, c);
      const uint64_t nm2 = f2pack(-msub, -msub);
      uint32_t pk[BN / 2];
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < BN; e += 2) {
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
      }
      {
        const uint64_t s2 = f2add(f2add(acc2[0], acc2[1]), f2add(acc2[2], acc2[3]));
        float s0, s1;
        f2unpack(s2, s0, s1);
        l = l * alpha + (s0 + s1);
      }
      TM_PH(3);
      TM_SM_EV(EV_EXP_DONE);
      // O is rescaled only when a row of this warp raised its running max.
      // Then PV_{j-1} must have completed: o_done has finished phase j-2 at
      // least (S_j completed after PV_{j-2}), so waiting for phase j-1 by
      // parity is unambiguous even though earlier phases were not waited on.
      TM_SM_EV(EV_O_READY);
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!mbar_wait(bar(C_ODONE + t), (j - 1) & 1, p.err, abort_flag)) ok = false;
        tc_fence_after();
        __syncwarp();
        {
          TM_SM_EV(EV_RESCALED);
          uint32_t o[D];
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_ld32p(o_addr + cc * 32, o + cc * 32);
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
          for (int cc = 0; cc < D / 32; ++cc) tmem_st32p(o_addr + cc * 32, o + cc * 32);
        }
      }
      TM_PH(4);
      __syncwarp();
#pragma unroll
      for (int cc = 0; cc < BN / 64; ++cc) tmem_st32p(s_addr + cc * 32, pk + cc * 32);
      tmem_wait_st();
      tc_fence_before();
      if (DUAL) {
        named_bar_arrive(NB_P + t, 160);   // P_t(j) stored: hand it to issuer t
        if (t == 0 && j == 0 && ti[1].nJ > 0) named_bar_arrive(NB_START, 160);
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C_PFULL + t));   // the wait helper hands it to the issuer
      }
      TM_PH(5);
      TM_SM_EV(EV_P_RELEASED);
    }
    }
#ifdef TM_PHASES
    if (tracer && blockIdx.x == g_tm_trace_block)
      for (int i = 0; i < 8; ++i) g_tm_trace[t][TM_TRACE_EVENTS - 8 + i] = static_cast<unsigned long long>(tm_ph[i]);
#endif
    // ---- epilogue
    bool have_o = false;
    if (ok && T.nJ > 0) {
      // chunked mode: two P.V may still be in flight, so wait for the
      // issuer's final commit instead of a P.V phase
      if (CH) have_o = mbar_wait(bar(C_DRAIN + t), 0, p.err, abort_flag);
      else have_o = mbar_wait(bar(C_ODONE + t), (T.nJ - 1) & 1, p.err, abort_flag);
      tc_fence_after();
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    __syncwarp();
    uint32_t o[D];
    if (__all_sync(0xffffffffu, have_o)) {
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32p(o_addr + cc * 32, o + cc * 32);
      tmem_wait_ld_regs<D>(o);
    } else {
#pragma unroll
      for (int e = 0; e < D; ++e) o[e] = 0u;
    }
    if (row_ok) {
      __half* orow = p.out + (T.row0 + r) * p.out_st + static_cast<int64_t>(h) * p.out_sh;
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

std::mutex g_mu2;

// One-time kernel attributes; the warpgroup register split assumes exactly
// LAUNCH_REGS per thread at launch (any other allocation could leave
// setmaxnreg.inc waiting), so a build that differs is refused.
template <int D, bool DUAL, bool CH, bool CACHE = false, bool F8 = false, bool TOKS = false>
tm_status prepare_pair_kernel() {
  using C = Cfg2<D, CACHE, TOKS>;
  static bool attr_done = false;
  std::lock_guard<std::mutex> lk(g_mu2);
  if (attr_done) return TM_OK;
  auto kern = attn_pair_kernel<D, TM_EXP2_EMU_PAIRS, DUAL, CH, CACHE, F8, TOKS>;
  cudaFuncAttributes fa;
  tm_status st = check_cuda(cudaFuncGetAttributes(&fa, kern));
  if (st != TM_OK) return st;
  if (fa.numRegs != C::LAUNCH_REGS) return TM_ERR_UNSUPPORTED;
  st = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  if (st != TM_OK) return st;
  attr_done = true;
  return TM_OK;
}

// Key tiles from which the two query tiles of a CTA get one tcgen05 issuer
// each.  With short rows of key tiles the single shared issuer measured
// faster (its fixed issue order keeps the tiles' softmax phases
// alternating); with long rows one issuer per tile removes the wait of each
// tile's P.V and next S behind the other tile's MMAs.
constexpr int64_t kDualIssuerKeyTiles = 64;

// With one issuer per query tile (d = 128), 64-key chunks alternating
// between two score slots per tile (chunked mode) instead of one 128-key
// score tile: the next chunk's QK^T is computed while the softmax works on
// the current one, so the softmax alone sets the pace.  Measured on B200
// (routing sweep, L = 16384): +2.5 % on all-FP16 launches, but -8 % at 68 %
// INT8 pairs, where the softmax's int32 -> fp32 conversion is no longer
// offset by the shorter INT8 QK^T on the chain.  Chunked mode is therefore
// used for launches without a routing bitmask only (0 disables it).
#ifndef TM_PAIR_CHUNKED
#define TM_PAIR_CHUNKED 1
#endif

// F8: q / k carry the FP8 E4M3 codes and tile scales in their codes / scales
// fields and bitmask is the FP8 bit plane (d = 128).  TOKS: k carries the
// INT8 cache's K codes (its scales field unused), k / v the cache's fp16 view,
// and the INT8 route's key scales are per token, from kst_ws laid out
// [Hkv][kst_tiles][128] fp32 (d = 128, bitmask non-null).
template <int D, bool F8 = false, bool TOKS = false>
tm_status launch_pair(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                      const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                      const uint32_t* bitmask,
                      int64_t mask_hs, int32_t g, int32_t causal, cudaStream_t stream,
                      const float* kst_ws = nullptr, int64_t kst_tiles = 0) {
  using C = Cfg2<D>;
  const int64_t maxk_tiles = ((cu ? max_k : k->T) + 127) / 128;
  const bool dual = maxk_tiles >= kDualIssuerKeyTiles;
  const bool chunked = !F8 && !TOKS && dual && D == 128 && TM_PAIR_CHUNKED && bitmask == nullptr;
  tm_status st = chunked ? prepare_pair_kernel<D, true, true>()
                         : (dual ? prepare_pair_kernel<D, true, false, false, F8, TOKS>()
                                 : prepare_pair_kernel<D, false, false, false, F8, TOKS>());
  if (st != TM_OK) return st;
  CUtensorMap mQ16, mQ8, mK16, mK8, mV16;
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
    st = encode_thd_map(&mQ8, q->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->T, q->H, D, q->H * D, D, D,
                        128, swz8);
    if (st != TM_OK) return st;
    st = encode_thd_map(&mK8, k->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k->T, k->H, D, k->H * D, D, D,
                        128, swz8);
    if (st != TM_OK) return st;
  } else {
    mQ8 = mQ16;
    mK8 = mK16;
  }
  Params2 p = {};
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
  p.g = g;
  p.causal = causal ? 1 : 0;
  p.batch = cu ? batch : 1;
  const int64_t maxq = cu ? max_q : q->T;
  const int64_t maxk = cu ? max_k : k->T;
  p.max_lk = maxk;
  p.n_qt_max = static_cast<int>((maxq + 127) / 128);
  p.n_pair_max = (p.n_qt_max + 1) / 2;
  p.W = tm_mask_words(maxk, 128, g);
  p.sched_zero = 0;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(D)));
  p.err = DevErr{device_error_word()};
  p.kst_ws = kst_ws;
  p.kst_tiles = kst_tiles;
  // KV heads per scheduling chunk: as many as keep their K / V (fp16 K, int8
  // K, fp16 V) within ~40 MB of L2, widened until a chunk fills two waves of
  // 148 CTAs; always a divisor of Hkv.
  {
    const double kv_bytes = static_cast<double>(maxk) * D * (2 + 1 + 2);
    int c = static_cast<int>(40.0e6 / (kv_bytes > 1.0 ? kv_bytes : 1.0));
    c = c < 1 ? 1 : (c > p.Hkv ? p.Hkv : c);
    while (c < p.Hkv && static_cast<int64_t>(c) * (p.Hq / p.Hkv) * p.batch * p.n_pair_max < 2 * 148) ++c;
    while (p.Hkv % c) ++c;
    p.kv_chunk = c;
  }
  const int64_t grid = static_cast<int64_t>(p.n_pair_max) * p.batch * p.Hq;
  if (grid == 0) return TM_OK;
  if (grid > 0x7fffffffLL) return TM_ERR_UNSUPPORTED;
  if (chunked)
    attn_pair_kernel<D, TM_EXP2_EMU_PAIRS, true, true, false>
        <<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mQ16, mQ8, mK16, mK8, mV16, p);
  else if (dual)
    attn_pair_kernel<D, TM_EXP2_EMU_PAIRS, true, false, false, F8, TOKS>
        <<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mQ16, mQ8, mK16, mK8, mV16, p);
  else
    attn_pair_kernel<D, TM_EXP2_EMU_PAIRS, false, false, false, F8, TOKS>
        <<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mQ16, mQ8, mK16, mK8, mV16, p);
  return check_cuda(cudaGetLastError());
}

// The INT8 K / V cache on the two-query-tile kernel (d = 128, 128-row query
// tiles, 128-key tiles): k and v carry codes [T, Hkv, 128] and fp16 scales
// [T, Hkv]; the routing bitmask and Q's INT8 codes and tile scales as for
// launch_pair.
tm_status launch_pair_cache(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                            const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                            const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                            cudaStream_t stream) {
  constexpr int D = 128;
  using C = Cfg2<D, true>;
  tm_status st = prepare_pair_kernel<D, true, false, true>();
  if (st != TM_OK) return st;
  CUtensorMap mQ16, mQ8, mK8, mV8;
  Params2 p = {};
  st = encode_thd_map(&mQ16, q->data, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, q->T, q->H, D, q->stride_t, q->stride_h,
                      64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mK8, k->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k->T, k->H, D, k->H * D, D, D, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  st = encode_thd_map(&mV8, v->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, v->T, v->H, D, v->H * D, D, D, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TM_OK) return st;
  if (bitmask != nullptr) {
    st = encode_thd_map(&mQ8, q->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->T, q->H, D, q->H * D, D, D, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != TM_OK) return st;
  } else {
    mQ8 = mQ16;
  }
  p.out = static_cast<__half*>(out->data);
  p.out_st = out->stride_t;
  p.out_sh = out->stride_h;
  p.q_scales = static_cast<const float*>(q->scales);
  p.k_scales = nullptr;
  p.bitmask = bitmask;
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
  p.n_pair_max = (p.n_qt_max + 1) / 2;
  p.W = tm_mask_words(maxk, 128, g);
  p.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(D)));
  p.err = DevErr{device_error_word()};
  p.sched_zero = 0;
  p.k_tok_scale = static_cast<const __half*>(k->scales);
  p.v_tok_scale = static_cast<const __half*>(v->scales);
  // KV heads per scheduling chunk, as in launch_pair, from the cache's bytes
  // per key row (codes of K and V)
  {
    const double kv_bytes = static_cast<double>(maxk) * D * 2;
    int c = static_cast<int>(40.0e6 / (kv_bytes > 1.0 ? kv_bytes : 1.0));
    c = c < 1 ? 1 : (c > p.Hkv ? p.Hkv : c);
    while (c < p.Hkv && static_cast<int64_t>(c) * (p.Hq / p.Hkv) * p.batch * p.n_pair_max < 2 * 148) ++c;
    while (p.Hkv % c) ++c;
    p.kv_chunk = c;
  }
  const int64_t grid = static_cast<int64_t>(p.n_pair_max) * p.batch * p.Hq;
  if (grid == 0) return TM_OK;
  if (grid > 0x7fffffffLL) return TM_ERR_UNSUPPORTED;
  attn_pair_kernel<D, TM_EXP2_EMU_PAIRS, true, false, true>
      <<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(mQ16, mQ8, mQ16, mK8, mV8, p);
  return check_cuda(cudaGetLastError());
}

}  // namespace

tm_status launch_attn_pair_cache(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                                 const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q,
                                 int32_t max_k, const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                                 cudaStream_t stream) {
  return launch_pair_cache(q, k, v, out, cu, cu_k, batch, max_q, max_k, bitmask, mask_hs, g, causal, stream);
}

tm_status launch_attn_pair_toks(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                                const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                                const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                                const float* kst_ws, int64_t kst_tiles, cudaStream_t stream) {
  if (q->d != 128 || bitmask == nullptr || kst_ws == nullptr) return TM_ERR_UNSUPPORTED;
  return launch_pair<128, false, true>(q, k, v, out, cu, cu_k, batch, max_q, max_k, bitmask, mask_hs, g, causal,
                                       stream, kst_ws, kst_tiles);
}

tm_status launch_attn_pair_fp8(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                               const int32_t* cu, int32_t batch, int32_t max_q, const uint32_t* bitmask_fp8,
                               int64_t mask_hs, int32_t g, int32_t causal, cudaStream_t stream) {
  if (q->d != 128) return TM_ERR_UNSUPPORTED;
  return launch_pair<128, true>(q, k, v, out, cu, nullptr, batch, max_q, max_q, bitmask_fp8, mask_hs, g, causal,
                                stream);
}

tm_status launch_attn_pair(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                           const int32_t* cu, const int32_t* cu_k, int32_t batch, int32_t max_q, int32_t max_k,
                           const uint32_t* bitmask, int64_t mask_hs, int32_t g, int32_t causal,
                           cudaStream_t stream) {
  if (q->d == 128)
    return launch_pair<128>(q, k, v, out, cu, cu_k, batch, max_q, max_k, bitmask, mask_hs, g, causal, stream);
  return launch_pair<64>(q, k, v, out, cu, cu_k, batch, max_q, max_k, bitmask, mask_hs, g, causal, stream);
}

}  // namespace tmk
