/*
 * tm.h -- C ABI of libtm: tile-routed FP16/INT8 fused prefill attention for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (TileMix, Lattice paper page, abstract): the Lq x Lk score
 * matrix of scaled-dot-product attention is cut into hardware-aligned
 * tile_m x tile_n score tiles; one routing bit per (query tile, group of g
 * adjacent key tiles), packed into a compact bitmask, sends the group's scores
 * through an FP16 or an INT8 QK^T; both routes feed one online-softmax state
 * and one P.V accumulation; every legal group is computed, so no visible
 * query-key pair is dropped; grouped-query attention, variable-length batches
 * and INT8 key/value caches are supported.  With no bitmask the call is plain
 * fused attention (MLX PR "Nax Refactor", attention tables: fp16, GQA,
 * causal).
 *
 * Conventions shared by every call
 *  - Tensors are token-major [T, H, d] ("THD"): element (t, h, c) is at
 *    data[t * stride_t + h * stride_h + c]; the innermost dimension is
 *    contiguous; strides are in elements.  d is 64 or 128.
 *  - Pointers are device pointers unless the argument name ends in _host.
 *    The caller owns every buffer.  The library allocates no device memory;
 *    it keeps only a per-process table of kernel attributes.
 *  - Every call is asynchronous on `stream` (a cudaStream_t / CUstream passed
 *    as void*, NULL = legacy default stream) and never synchronises, except
 *    tm_get_device_error.
 *  - Arguments are validated on the host before any launch; a rejected call
 *    launches nothing and returns TM_ERR_INVALID_ARG or TM_ERR_UNSUPPORTED.
 *    A failed launch returns TM_ERR_CUDA (tm_last_cuda_error() gives the CUDA
 *    code).  Conditions only the device can see (a sequence longer than
 *    max_seqlen; a pipeline wait that exceeded its time limit) are recorded
 *    in a device error word read by tm_get_device_error.
 *  - Variable-length batches: cu_seqlens is a device int32 array [batch + 1],
 *    non-decreasing, cu_seqlens[0] = 0; sequence b holds rows
 *    cu_seqlens[b] .. cu_seqlens[b+1]-1 of BOTH Q and K/V (self-attention
 *    prefill), so Lq = Lk = its length.  max_seqlen must be >= every length.
 *    With cu_seqlens == NULL there is one sequence, Lq = q->T, Lk = k->T,
 *    and batch / max_seqlen are ignored.
 *  - Tiles restart at every sequence.  Query tile I of sequence b is global
 *    query tile I_glob = (number of query tiles of sequences < b) + I; key
 *    tiles are numbered the same way with tile_n.
 *  - Causal masking is bottom-right aligned: key j is visible to query i iff
 *    j < Lk and j <= i + Lk - Lq.  A query row with no visible key is 0.
 */
#ifndef TM_H_
#define TM_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TM_OK = 0,
  TM_ERR_INVALID_ARG = 1,  /* bad pointer, shape, stride, alignment or length */
  TM_ERR_UNSUPPORTED = 2,  /* valid request outside what is built (d, tiles) */
  TM_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  TM_ERR_TIMEOUT = 4       /* a device pipeline wait exceeded its limit */
} tm_status;

/* How a tensor's INT8 scales are laid out (field tm_tensor.scale_kind). */
typedef enum {
  TM_SCALE_NONE = 0,
  TM_SCALE_TILE = 1,   /* fp32 [n_tiles, H]: one scale per (tile, head), written by tm_quantize_qk */
  TM_SCALE_TOKEN = 2   /* fp16 [T, H]: one scale per (token, head), an INT8 K/V cache */
} tm_scale_kind;

/* One attention operand or output, [T, H, d].
 *  data     fp16 values with strides stride_t / stride_h (elements); for an
 *           INT8 cache operand (scale_kind == TM_SCALE_TOKEN) data is NULL.
 *  codes    int8 values, dense [T, H, d] (stride_t = H*d, stride_h = d), or NULL.
 *  scales   see scale_kind, or NULL.
 * Alignment: data and codes 16-byte aligned; stride_t and stride_h multiples
 * of 8 elements; scales 4-byte (fp32) or 2-byte (fp16) aligned. */
typedef struct {
  void* data;
  int64_t T, H, d;
  int64_t stride_t, stride_h;
  const int8_t* codes;
  const void* scales;
  int32_t scale_kind;
} tm_tensor;

/* ---------------------------------------------------------------------------
 * tm_quantize_qk -- per-tile symmetric INT8 quantisation of Q and K.
 *
 * TileMix abstract: the INT8 route computes scores from INT8 codes.  The
 * per-tile rule (symmetric absmax / 127) is the one this library fixes:
 *   amax = max |x| over the tile's rows x d of one head (tiles of tile_m rows
 *          for Q, tile_n rows for K, restarting at every sequence);
 *   s    = fl32(amax / 127)                  (IEEE fp32 division)
 *   code = clamp(rne(fl32(x / s)), -127, 127), and all codes 0 when s == 0.
 * q: fp16 [Tq, Hq, d] (its codes/scales fields are ignored); q_codes: int8
 * dense [Tq, Hq, d]; q_scales: fp32 [n_qtiles, Hq].  Same for k with tile_n
 * into k_codes [Tk, Hkv, d] / k_scales [n_ktiles, Hkv]; k may be NULL (Q only;
 * used with an INT8 K/V cache).  Code rows outside every sequence are not
 * written.  tile_m, tile_n in {64, 128}.  A sequence of more than 65535
 * tiles (over 8.3 M rows at 128-row tiles) returns TM_ERR_UNSUPPORTED.
 * Results are bit-identical to the definition above (no contraction of the
 * division, round-to-nearest-even conversion).
 * ------------------------------------------------------------------------- */
tm_status tm_quantize_qk(const tm_tensor* q, const tm_tensor* k,
                         int8_t* q_codes, float* q_scales,
                         int8_t* k_codes, float* k_scales,
                         const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen,
                         int32_t tile_m, int32_t tile_n, void* stream);

/* tm_quantize_qk with separate key offsets (prefix-cached prefill): Q tiles
 * restart at every cu_seqlens_q[b], K tiles at every cu_seqlens_k[b]; the
 * sequence's lq new queries attend to its lk keys.  max_seqlen_q / _k bound
 * the per-sequence lengths.  Scales are written per side in tile order over
 * all sequences ([n_qtiles, Hq] and [n_ktiles, Hkv]; tm_count_tiles with the
 * side's offsets).  TM_ERR_INVALID_ARG when an offset array is null or a
 * maximum is not positive; otherwise as tm_quantize_qk. */
tm_status tm_quantize_qk_varlen(const tm_tensor* q, const tm_tensor* k, int8_t* q_codes, float* q_scales,
                                int8_t* k_codes, float* k_scales, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k, int32_t batch, int32_t max_seqlen_q,
                                int32_t max_seqlen_k, int32_t tile_m, int32_t tile_n, void* stream);

/* FP8 E4M3 codes of the third precision (the pages name FP16 and INT8; the
 * "Add rowwise scaling to Float8Inference module" page, Summary, describes
 * fp8 operands with per-tensor or per-axis scales).  Per (head, tile) as in
 * tm_quantize_qk, with s = fl32(amax / 448) (448: the largest finite E4M3
 * value) and code = E4M3 round-to-nearest-even of fl32(x / s), saturating at
 * +-448 (bit 7 sign, bits 6..3 exponent with bias 7, bits 2..0 mantissa;
 * a negative value that rounds to zero gives the code of -0); amax == 0
 * gives s = 0 and codes 0.  Layouts, arguments and errors as
 * tm_quantize_qk, codes as uint8.  Bit-identical to the definition. */
tm_status tm_quantize_qk_fp8(const tm_tensor* q, const tm_tensor* k, uint8_t* q_codes, float* q_scales,
                             uint8_t* k_codes, float* k_scales, const int32_t* cu_seqlens, int32_t batch,
                             int32_t max_seqlen, int32_t tile_m, int32_t tile_n, void* stream);

/* ---------------------------------------------------------------------------
 * Routing bitmask layout (TileMix abstract: routing decisions packed into a
 * bitmask, one bit per query tile x key-tile group, a group being several
 * neighbouring key tiles).
 *   word  bitmask[h * mask_head_stride + I_glob * W + G / 32], bit G % 32;
 *   G = J / g is the group of key tile J;  bit 1 = INT8, 0 = FP16;
 *   W = tm_mask_words(max Lk, tile_n, g) = ceil(ceil(ceil(Lk/tile_n)/g)/32).
 * Bits of groups with no visible pair for the query tile are ignored.
 * A per-head mask has mask_head_stride = n_qtiles * W; 0 shares one plane.
 * ------------------------------------------------------------------------- */
int32_t tm_mask_words(int64_t max_lk, int32_t tile_n, int32_t g);

/* Number of tiles of `tile` rows over a batch: sum_b ceil(len_b / tile) from
 * a HOST copy of cu_seqlens, or ceil(L / tile) when cu_seqlens_host == NULL.
 * Returns -1 on invalid arguments. */
int64_t tm_count_tiles(const int32_t* cu_seqlens_host, int32_t batch, int64_t L, int32_t tile);

/* ---------------------------------------------------------------------------
 * tm_build_mask -- seeded routing bitmask on the device.
 *
 * The pages say only that routing is decided per tile group at inference
 * time without training.  This builder draws an independent Bernoulli(p)
 * per group: for head h (0..Hq-1), query tile I_glob, group G that is legal
 * (holds a visible pair for the tile) and not forced,
 *   u   = (splitmix64(seed XOR (h * 2^40 + I_glob * 2^20 + G)) >> 11) * 2^-53
 *   bit = (u < p)
 * where splitmix64(x) is the SplitMix64 output function applied to
 * x + 0x9E3779B97F4A7C15.  Forced groups are 0: with force_diag the group that
 * holds the query tile's last visible key tile, with force_sink group 0.
 * Illegal groups and padding bits are 0.  Writes the n_qtiles * W words of
 * every head plane h at bitmask + h * mask_head_stride, where n_qtiles =
 * tm_count_tiles(cu_seqlens_host, batch, Lq, tile_m) and W = tm_mask_words(
 * max Lk, tile_n, g); mask_head_stride >= n_qtiles * W is the caller's
 * contract (checked on the host when cu_seqlens == NULL).
 * Lq, Lk: lengths when cu_seqlens == NULL; max_seqlen: bound when not.
 * Hq < 2^24, n_qtiles < 2^20, groups < 2^20; 0 <= p <= 1.
 * ------------------------------------------------------------------------- */
tm_status tm_build_mask(uint32_t* bitmask, int32_t Hq,
                        const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen,
                        int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n, int32_t g,
                        int32_t causal, double p, uint64_t seed,
                        int32_t force_diag, int32_t force_sink, int64_t mask_head_stride,
                        void* stream);

/* tm_build_mask with separate key offsets: sequence b has lq = cu_q[b+1] -
 * cu_q[b] queries and lk = cu_k[b+1] - cu_k[b] keys, bottom-right causal;
 * W = tm_mask_words(max_seqlen_k, tile_n, g).  A key sequence longer than
 * max_seqlen_k is reported by tm_get_device_error (TM_ERR_INVALID_ARG) and
 * its rows are not written. */
tm_status tm_build_mask_varlen(uint32_t* bitmask, int32_t Hq, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, int32_t batch, int32_t max_seqlen_q,
                               int32_t max_seqlen_k, int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                               double p, uint64_t seed, int32_t force_diag, int32_t force_sink,
                               int64_t mask_head_stride, void* stream);

/* Content-driven routing bitmask (the frontier policy; the pages adjust
 * precision during inference but give no policy).  Same layout, legality and
 * forcing as tm_build_mask.  With symmetric absmax/127 codes the INT8 score
 * of a tile pair differs from the fp16 score by at most
 * d * s_q * s_k * (127 + 1/4); group G of query tile I (head h, kv head
 * h / (Hq / Hkv)) is routed INT8 iff fl32(s_q[I, h] * mk) <= tau, where mk is
 * the largest s_k over the group's key tiles that I sees.  tau = +inf routes
 * every eligible group INT8, tau < 0 none.
 *   q_scales: device fp32 [n_qtiles, Hq], k_scales: device fp32 [n_ktiles, Hkv]
 *             (the tile scales written by tm_quantize_qk).
 *   Other arguments as for tm_build_mask.  TM_ERR_INVALID_ARG for Hq % Hkv
 *   != 0, a NaN tau, null scales or the conditions of tm_build_mask. */
tm_status tm_build_mask_scale_policy(uint32_t* bitmask, int32_t Hq, int32_t Hkv, const int32_t* cu_seqlens,
                                     int32_t batch, int32_t max_seqlen, int64_t Lq, int64_t Lk, int32_t tile_m,
                                     int32_t tile_n, int32_t g, int32_t causal, const float* q_scales,
                                     const float* k_scales, float tau, int32_t force_diag, int32_t force_sink,
                                     int64_t mask_head_stride, void* stream);

/* tm_build_mask_scale_policy with separate key offsets (prefix-cached
 * prefill): sequence b has lq = cu_q[b+1] - cu_q[b] queries and lk =
 * cu_k[b+1] - cu_k[b] keys, bottom-right causal; key tiles are numbered per
 * key sequence (k_scales: device fp32 [sum_b ceil(lk_b / tile_n), Hkv], as
 * tm_quantize_qk writes them with key offsets, or as tm_key_tile_scales
 * writes them from an INT8 cache); W = tm_mask_words(max_seqlen_k, tile_n, g).
 * A key sequence longer than max_seqlen_k is reported by tm_get_device_error
 * (TM_ERR_INVALID_ARG) and its rows are not written.  TM_ERR_INVALID_ARG for
 * a null cu_seqlens_q / cu_seqlens_k, max_seqlen_k <= 0 or the conditions of
 * tm_build_mask_scale_policy. */
tm_status tm_build_mask_scale_policy_varlen(uint32_t* bitmask, int32_t Hq, int32_t Hkv,
                                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                            int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                            int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                                            const float* q_scales, const float* k_scales, float tau,
                                            int32_t force_diag, int32_t force_sink, int64_t mask_head_stride,
                                            void* stream);

/* Key-tile statistic of the scale policy for an INT8 cache, whose keys carry
 * one fp16 scale per token and kv head.  For the cache the FP16 route reads
 * k^ = fp16(c_k * s_k) and the INT8 route s_q * s_k * (c_q . c_k), so a score's
 * two values differ by at most about d * s_q * s_k * (127/2 + 127^2 / 2^11):
 * again s_q times the key's scale.  This writes, per key tile J and kv head
 * hk, the largest token scale over the tile's tokens, as fp32 (exact); fed to
 * tm_build_mask_scale_policy(_varlen) as k_scales, each group's statistic is
 * then the largest token scale over its visible key tiles' tokens.
 *   k_tile_scales: device fp32 [n_ktiles, Hkv] (out), key tiles numbered per
 *                  sequence in order, each sequence starting a new tile.
 *   k_token_scales: device fp16 [Tk, Hkv], contiguous (the cache's K scales),
 *                  finite and >= 0.
 *   cu_seqlens_k: device int32 [batch+1] key offsets, or NULL for one
 *                  sequence of Lk keys; max_seqlen_k bounds the key lengths
 *                  (a longer sequence is reported by tm_get_device_error and
 *                  not written).
 * TM_ERR_INVALID_ARG for null or misaligned pointers, Hkv <= 0, tile_n <= 0,
 * batch <= 0 with offsets, negative lengths. */
tm_status tm_key_tile_scales(float* k_tile_scales, const void* k_token_scales, int32_t Hkv,
                             const int32_t* cu_seqlens_k, int32_t batch, int32_t max_seqlen_k, int64_t Lk,
                             int32_t tile_n, void* stream);

/* Same bits computed on the host (bitmask_host and cu_seqlens_host are host
 * pointers), written with mask_head_stride = n_qtiles * W; bit-identical to
 * tm_build_mask. */
tm_status tm_build_mask_host(uint32_t* bitmask_host, int32_t Hq,
                             const int32_t* cu_seqlens_host, int32_t batch,
                             int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n, int32_t g,
                             int32_t causal, double p, uint64_t seed,
                             int32_t force_diag, int32_t force_sink);

/* Host statistics of a host bitmask: n_vis = visible query-key pairs summed
 * over heads and sequences; e8 = those in INT8-routed tiles.  The realised
 * INT8 fraction is e8 / n_vis.  bitmask_host may be NULL (e8 = 0). */
tm_status tm_route_stats(const uint32_t* bitmask_host, int64_t mask_head_stride, int32_t Hq,
                         const int32_t* cu_seqlens_host, int32_t batch,
                         int64_t Lq, int64_t Lk, int32_t tile_m, int32_t tile_n, int32_t g,
                         int32_t causal, double* n_vis, double* e8);

/* tm_route_stats with separate (host) key offsets per sequence. */
tm_status tm_route_stats_varlen(const uint32_t* mask_host, int64_t mask_head_stride, int32_t Hq,
                                const int32_t* cu_seqlens_q_host, const int32_t* cu_seqlens_k_host, int32_t batch,
                                int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal, double* n_vis,
                                double* e8);

/* ---------------------------------------------------------------------------
 * tm_attn_fwd -- fused tile-routed attention forward (prefill).
 *
 * For every sequence, query head h (KV head h / (Hq / Hkv)) and visible pair
 * (i, j) in query tile I_glob and key tile J:
 *   FP16 route: S_ij = sigma * q_i . k_j                 (fp16 operands)
 *   INT8 route: S_ij = sigma * s_q * s_k * (cq_i . ck_j) (int8 operands,
 *               exact int32 sum; s_q = q tile scale, s_k = k tile scale or,
 *               for an INT8 cache, the scale of key j)
 *   sigma = 1/sqrt(d); route = bit of group J / g (always FP16 when bitmask
 *   is NULL); out_i = fp16( sum_j softmax_j(S_i.) v_j ) with P rounded to fp16
 *   for the P.V product, fp32 accumulation and fp32 row sums.
 *
 * q:   fp16 data [Tq, Hq, d]; when bitmask != NULL also codes and
 *      TM_SCALE_TILE scales (from tm_quantize_qk with the same tile_m).
 * k,v: either fp16 data [Tk, Hkv, d] (k also with codes + TM_SCALE_TILE scales
 *      from tm_quantize_qk with tile_n when bitmask != NULL), or an INT8 cache:
 *      data NULL, codes + TM_SCALE_TOKEN scales, for BOTH k and v.  The cache
 *      is dequantised to fp16 (fp16(code * scale)) in shared memory for FP16
 *      groups and for all of V; INT8 groups use the K codes directly.
 * out: fp16 data [Tq, Hq, d]; every row of every sequence is written.
 * bitmask / mask_head_stride: see the layout above; NULL = all FP16.
 * tile_m in {64, 128}; tile_n in {64, 128}; g >= 1; d in {64, 128};
 * Hq % Hkv == 0; the INT8 cache requires d == 128 and tile_n == 128.
 * ------------------------------------------------------------------------- */
tm_status tm_attn_fwd(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                      const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen,
                      const uint32_t* bitmask, int64_t mask_head_stride,
                      int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal, void* stream);

/* tm_attn_fwd with separate key offsets (prefix-cached prefill, also over an
 * INT8 K/V cache): sequence b's queries are rows cu_seqlens_q[b] .. of q and
 * out, its keys rows cu_seqlens_k[b] .. of k and v (or of the cache), and
 * query i of a sequence sees key j iff j < lk and (not causal or
 * j <= i + lk - lq).  The bitmask is laid out as by tm_build_mask_varlen and
 * the tile scales as by tm_quantize_qk_varlen.  A key sequence longer than
 * max_seqlen_k is reported by tm_get_device_error (TM_ERR_INVALID_ARG); its
 * query rows are not written.  Otherwise as tm_attn_fwd. */
tm_status tm_attn_fwd_varlen(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
                             int32_t max_seqlen_q, int32_t max_seqlen_k, const uint32_t* bitmask,
                             int64_t mask_head_stride, int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                             void* stream);

/* ---------------------------------------------------------------------------
 * tm_attn_fwd_cache_ws -- tm_attn_fwd / tm_attn_fwd_varlen over an INT8 K/V
 * cache, with the cache expanded once per call into a caller-owned workspace.
 *
 * TileMix (Lattice paper page, abstract) supports INT8 K/V caches; the
 * FP16-routed groups and P.V read the cache's fp16 view fp16(code * scale)
 * and the INT8-routed groups its K codes with the scale of each key.  Every
 * K / V tile of a KV head is read by every query tile of the Hq / Hkv query
 * heads of its group, so this call first writes the fp16 view of K and V
 * (and the per-token K scales as fp32, one row of 128 per key tile) into `workspace`
 * with one HBM-bound pass, then runs the attention on that view.  Results
 * equal tm_attn_fwd's over the same cache (same scores, same softmax).
 *   k, v: the INT8 cache (data NULL, codes [Tk, Hkv, 128] dense int8 +
 *         TM_SCALE_TOKEN fp16 scales [Tk, Hkv] dense), as for tm_attn_fwd.
 *   cu_seqlens_q: NULL for one sequence (Lq = q->T, Lk = k->T); else the
 *         query offsets, with cu_seqlens_k the key offsets or NULL (keys use
 *         the query offsets); max_seqlen_q / max_seqlen_k as for
 *         tm_attn_fwd_varlen.
 *   workspace: device memory of at least tm_cache_workspace_bytes(Tk, Hkv,
 *         batch) bytes (batch = 0 without cu_seqlens_q), 256-byte aligned,
 *         owned by the caller; overwritten by each call and free again once
 *         the call's work on `stream` has finished.
 * 128 x 128 tiles, d = 128.  tile_m = 64 runs tm_attn_fwd's in-kernel
 * conversion and leaves the workspace untouched.  TM_ERR_INVALID_ARG for a
 * null or short workspace, k / v that are not a cache, or the conditions of
 * tm_attn_fwd(_varlen).
 * ------------------------------------------------------------------------- */
int64_t tm_cache_workspace_bytes(int64_t Tk, int32_t Hkv, int32_t batch);
tm_status tm_attn_fwd_cache_ws(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
                               int32_t max_seqlen_q, int32_t max_seqlen_k, const uint32_t* bitmask,
                               int64_t mask_head_stride, int32_t tile_m, int32_t tile_n, int32_t g, int32_t causal,
                               void* workspace, int64_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * tm_attn_fwd_routed_noalloc -- the routed prefill step for callers that
 * cannot allocate device memory.  (Library addition; it has no counterpart
 * in the paper.)
 *
 * Some callers cannot give the library scratch buffers: a serving engine that
 * reserves nearly all device memory for its own pools at start-up and has no
 * allocator to lend to a C library, or a deployment that forbids cudaMalloc
 * after initialisation because it may synchronise the device and has
 * unbounded latency.  This call runs tm_quantize_qk, tm_build_mask and
 * tm_attn_fwd for one sequence (no cu_seqlens; Lq = q->T, Lk = k->T) with the
 * INT8 codes, tile scales and routing mask placed in a fixed device array that
 * the library owns: TM_NOALLOC_SCRATCH_BYTES on every GPU that loads the
 * library, held until the process exits.  The caller passes q, k, v (fp16
 * data; their codes / scales fields are ignored) and out, as for tm_attn_fwd,
 * and the routing parameters of tm_build_mask (mask_head_stride is implied).
 * No cudaMalloc, cudaFree or other allocating routine is called.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress)
 *    in the current device's context, so a reset device or another context
 *    gets its own address; the lookup allocates nothing.  The first call on a
 *    device also sets up the library's module there: make it before any
 *    stream capture.
 *  - Every argument is checked before the lookup and before any launch, so a
 *    rejected call leaves the array and out untouched.  The codes / scales
 *    fields of q, k and v are ignored (v is read as fp16 values).
 *  - All calls share the array and it keeps the last call's contents; every
 *    byte a call reads it first writes, so nothing needs clearing.  Calls
 *    that overlap on the GPU (other streams, other host threads on the same
 *    device) race on the array: serialise them.
 *  - A problem whose codes, scales and mask need more than
 *    TM_NOALLOC_SCRATCH_BYTES (about Lq*Hq*d + Lk*Hkv*d bytes) returns
 *    TM_ERR_UNSUPPORTED before any launch.
 * ------------------------------------------------------------------------- */
#define TM_NOALLOC_SCRATCH_BYTES (32u << 20)
tm_status tm_attn_fwd_routed_noalloc(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v,
                                     tm_tensor* out, int32_t tile_m, int32_t tile_n, int32_t g,
                                     int32_t causal, double p, uint64_t seed,
                                     int32_t force_diag, int32_t force_sink, void* stream);

/* Reads and clears the device error word after synchronising `stream`.
 * Returns TM_OK, TM_ERR_TIMEOUT (a pipeline wait gave up; the output of the
 * affected call is unspecified) or TM_ERR_INVALID_ARG (a sequence exceeded
 * max_seqlen; its extra tiles were not computed). */
tm_status tm_get_device_error(void* stream);

/* Failure-detection self-test: launches one thread that waits, with the
 * library's bounded mbarrier wait, on a barrier nothing arrives on, giving up
 * after limit_ns (1 ns .. 10 s) of GPU global time.  The wait records a
 * timeout in the device error word, so a following tm_get_device_error
 * returns TM_ERR_TIMEOUT (and clears it); the context stays usable.  Nothing
 * faults, traps or hangs. */
tm_status tm_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Instruction-rate probes behind the kernels' secondary bounds (a
 * measurement utility; the pages have no counterpart).  On the current
 * device, writes out[0..4]:
 *   out[0]  MUFU ex2.approx.f32, SM-clock cycles per warp instruction per SM
 *           sub-partition (4 warps per sub-partition);
 *   out[1]  cvt.rn.f32.s32 (int32 -> fp32), same unit, one integer shift
 *           per value included;
 *   out[2]  the kernels' exact int32 -> fp32 conversion (integer add of the
 *           bits of 1.5 * 2^23, one fp32 subtract), cycles per value per
 *           sub-partition, one integer shift per value included;
 *   out[3]  tcgen05.mma kind::f16 M128 N128 K16, cycles per MMA on one SM,
 *           issued back to back;
 *   out[4]  tcgen05.mma kind::i8 M128 N128 K32, same.
 * A tensor probe whose bounded wait expired reports -1.
 * scratch: caller-owned device memory of at least tm_probe_scratch_bytes()
 * bytes, 16-byte aligned (the probe allocates nothing).  Synchronises
 * `stream` (a cudaStream_t) before returning.  TM_ERR_INVALID_ARG for a
 * null or short buffer or n_out < 5. */
int64_t tm_probe_scratch_bytes(void);
tm_status tm_probe_rates(double* out, int32_t n_out, void* scratch, int64_t scratch_bytes, void* stream);

/* Attention with the FP8 third precision (the pages route between FP16 and
 * INT8; fp8 operands with per-axis scales: "Add rowwise scaling to
 * Float8Inference module" page, Summary).  As tm_attn_fwd with 128 x 128 tiles and
 * d = 128, plus a second routing bit plane `bitmask_fp8` in the layout of
 * `bitmask` (same mask_head_stride): a legal group whose INT8 bit is clear
 * and whose FP8 bit is set computes its scores from the E4M3 codes of
 * tm_quantize_qk_fp8, S_ij = sigma * s_q * s_k * (dot product of the decoded
 * codes), accumulated in fp32 by the tensor core (kind::f8f6f4); INT8 wins
 * when both bits are set.  bitmask may be NULL (no INT8 groups; then Q / K
 * need no INT8 codes).  q_fp8_codes [Tq, Hq, 128] / q_fp8_scales
 * [n_qtiles, Hq], k_fp8_codes [Tk, Hkv, 128] / k_fp8_scales [n_ktiles, Hkv]
 * as written by tm_quantize_qk_fp8 with the same tiles and cu_seqlens.
 * fp16 K / V only (no INT8 cache).  Codes 16-byte aligned, masks and scales
 * 4-byte aligned, else TM_ERR_INVALID_ARG; other d, tiles or a cache:
 * TM_ERR_UNSUPPORTED. */
tm_status tm_attn_fwd_fp8(const tm_tensor* q, const tm_tensor* k, const tm_tensor* v, tm_tensor* out,
                          const int32_t* cu_seqlens, int32_t batch, int32_t max_seqlen, const uint32_t* bitmask,
                          const uint32_t* bitmask_fp8, int64_t mask_head_stride, const uint8_t* q_fp8_codes,
                          const float* q_fp8_scales, const uint8_t* k_fp8_codes, const float* k_fp8_scales,
                          int32_t g, int32_t causal, void* stream);

/* Kernel choice for attention with 128 x 128 tiles (tm_attn_fwd,
 * tm_attn_fwd_varlen; fp16 K / V; d = 64 or 128).  Two kernels compute the
 * same result: one holding two 128-row query tiles per CTA (faster per tile
 * once INT8 tiles are routed at d = 128) and one holding a single query tile
 * per CTA with three score buffers in tensor memory (twice as many CTAs; at
 * d = 64 its two softmax warpgroups run independent streams over alternate
 * key tiles).  choice: 0 automatic (the default: at d = 64 the one-tile
 * kernel; at d = 128 the one-tile kernel when the two-tile kernel would
 * launch fewer CTAs than the GPU has SMs, except for an all-FP16 launch
 * without a causal mask that the two-tile kernel still spreads over at
 * least 80 % of the SMs in one wave, and for an all-FP16 launch without a
 * causal mask whose last wave it fills clearly better), 1 always the
 * two-tile kernel, 2 always the one-tile kernel.  Process-wide;
 * TM_ERR_INVALID_ARG for any other value. */
tm_status tm_set_attn_kernel(int32_t choice);

/* Which of the two kernels above tm_attn_fwd / tm_attn_fwd_varlen would run
 * for a launch with 128 x 128 tiles, fp16 K / V and no FP8 route (the pages
 * have no counterpart; a query for callers tuning their shapes).  max_q /
 * max_k: the longest query / key sequence; batch: sequences (1 without
 * offsets); hq: query heads; d: 64 or 128; routed: non-zero when a routing
 * bitmask is given; causal: non-zero for the bottom-right causal mask;
 * sm_count: the GPU's SM count, or 0 for the current device's (the only
 * case that queries the device).  Returns 1 for the two-query-tile kernel,
 * 2 for the one-query-tile kernel (honouring tm_set_attn_kernel), 0 for
 * invalid arguments.  Host-only: launches nothing. */
int32_t tm_attn_kernel_choice(int64_t max_q, int64_t max_k, int32_t batch, int32_t hq, int32_t d, int32_t routed,
                              int32_t causal, int32_t sm_count);

/* Head-sharded prefill: reassembly of the output after the all-gather.
 * The pages do not speak of more than one GPU.  Every step of the method
 * (TileMix abstract: per-tile quantisation, routing bits, scores, shared
 * online softmax) is computed per query head, and grouped-query heads (the
 * GQA shapes of the MLX PR "Nax Refactor" attention tables) share only their
 * K / V, so one problem shards over ranks by blocks of consecutive query
 * heads with no exchange on the data path: rank r computes heads head_start[r] ..
 * head_start[r+1]-1 of every token into the first head slots of its
 * [T, h_cap, d] slice, and an all-gather of those equal-size slices gives
 * `gathered`, fp16 [world, T, h_cap, d] contiguous.  This writes out[t, h, :]
 * = gathered[r, t, h - head_start[r], :] for the rank r owning h.
 *   out          device fp16 [T, Hq, d], heads contiguous (stride d), row
 *                stride out_stride_t elements (>= Hq*d, multiple of 8);
 *   head_start   HOST int32 [world+1]: head_start[0] = 0, non-decreasing,
 *                head_start[world] = Hq, every count <= h_cap;
 *   d            multiple of 8; world in 1..64; both pointers 16-byte aligned.
 * The two buffers must not overlap.  Asynchronous on `stream`; TM_ERR_INVALID_ARG
 * on any violated condition (nothing is launched); T = 0 is a no-op. */
tm_status tm_merge_head_shards(void* out, int64_t out_stride_t, const void* gathered, int64_t T, int32_t Hq,
                               int32_t d, int32_t world, int32_t h_cap, const int32_t* head_start, void* stream);

/* Static description of a status code. */
const char* tm_status_string(tm_status s);

/* CUDA error code of the last TM_ERR_CUDA returned on this thread (0 if none). */
int32_t tm_last_cuda_error(void);

/* Library version, "major.minor.patch". */
const char* tm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TM_H_ */
