"""Plain fp64 CPU oracle of tile-routed FP16/INT8 prefill attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

What is computed, and where it comes from
-----------------------------------------
TileMix (Lattice paper page "TileMix ..."), abstract:
  * the Lq x Lk score matrix is cut into tile_m x tile_n score tiles;
  * one routing bit covers g adjacent KEY tiles (a "group"); bits are packed
    into a compact bitmask, one bit per (query tile, key-tile group);
  * a group's scores are computed either from FP16 operands or from INT8
    codes; both feed the same (online) softmax state and the same P.V sum;
  * every legal group (one holding at least one visible query-key pair) is
    computed, so no visible pair is ever dropped;
  * grouped-query attention, variable-length batches and INT8 K/V caches.
MLX PR "Nax Refactor" (ml-explore/mlx #3271), attention tables: fused fp16
SDPA with GQA (n_qh / n_kvh columns) and causal masking; the near-equal
causal and non-causal times of its qsl=512 / ksl=4096 rows fix causal
alignment to the bottom-right corner.

The abstract leaves the numerics open.  The readings taken here (each one is
also listed with its reason in the design notes of this repository):
  (a) quantiser: symmetric per-tile absmax/127; scale s = fl32(amax / 127);
      code = clamp(rne(fl32(x / s)), -127, 127); amax == 0 gives s = 0 and
      all codes 0.  Q tiles are tile_m rows x d of one head, K tiles tile_n
      rows x d of one KV head; tiles restart at every sequence.
  (b) INT8 score = sigma * s_q * s_k * (integer dot product of the codes);
      with an INT8 K cache the key scale is the per-token cache scale.
  (c) sigma = 1/sqrt(d), applied after dequantisation.
  (d) bit 1 = INT8; an all-zero mask is plain attention.
  (e) groups run along keys; the last group of a row may be partial.
  (f) causal masking is bottom-right aligned: key j is visible to query i
      iff j < Lk and j <= i + Lk - Lq.
  (g) a group is legal iff it holds a visible pair for some row of the
      query tile; bits of illegal groups are ignored.
  (h) GQA: query head h reads KV head h // (Hq / Hkv).
  (j) variable-length batches share one cu_seqlens for Q and K
      (self-attention prefill); query and key tiles restart per sequence.
      With a separate cu_seqlens_k (prefix-cached prefill: each sequence's
      lq new queries attend to lk >= lq keys, prefix first), key rows of
      sequence b are cu_k[b] .. cu_k[b+1]-1 and causal masking stays
      bottom-right per sequence (reading (f) with that sequence's Lq, Lk).
  (k) a query row with no visible key outputs 0.
  (m) the mask builder draws an independent Bernoulli(p) per eligible group
      from a counter-based hash (splitmix64); the group holding the query
      tile's last visible key tile ("diagonal") and group 0 ("sink") can be
      forced to FP16.
  (p) a third precision (the TileMix abstract names FP16 and INT8 only;
      the "Add rowwise scaling to Float8Inference module" page, Summary,
      gives per-tensor and per-axis fp8 scales): FP8 E4M3 codes with a
      symmetric per-tile scale s = fl32(amax / 448) (448 is E4M3's largest
      finite value), code = E4M3 round-to-nearest-even of fl32(x / s),
      saturating at +-448; amax == 0 gives s = 0 and codes 0.  A second bit
      plane in the routing mask's layout selects FP8 for a group whose INT8
      bit is clear (two bits per group: INT8 wins when both are set).  FP8
      score = sigma * s_q * s_k * (exact dot product of the decoded codes).

Because online softmax is an exact rewrite of ordinary softmax, the oracle
computes ordinary softmax attention over the per-tile-routed scores in fp64
and does not emulate any streaming order.  Query rows are evaluated one query
tile at a time only to bound memory; every row is independent.
"""

from __future__ import annotations

import math

import numpy as np

SPLITMIX_GAMMA = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1


# --------------------------------------------------------------------------
# geometry: sequences, tiles, visibility
# --------------------------------------------------------------------------

def seq_table(Tq, Tk=None, cu_seqlens=None, cu_seqlens_k=None):
    """Sequences as (q_start, Lq, k_start, Lk).

    Without ``cu_seqlens`` there is one sequence with Lq = Tq, Lk = Tk (Tq and
    Tk may differ).  With ``cu_seqlens`` (reading (j)) sequence b spans rows
    cu[b] .. cu[b+1]-1 of both Q and K, so Lq = Lk = cu[b+1] - cu[b]; with
    ``cu_seqlens_k`` as well its keys are rows cu_k[b] .. cu_k[b+1]-1 of K.
    """
    if cu_seqlens is None:
        return [(0, int(Tq), 0, int(Tq if Tk is None else Tk))]
    cu = [int(c) for c in cu_seqlens]
    ck = cu if cu_seqlens_k is None else [int(c) for c in cu_seqlens_k]
    assert len(ck) == len(cu)
    return [(cu[b], cu[b + 1] - cu[b], ck[b], ck[b + 1] - ck[b]) for b in range(len(cu) - 1)]


def n_tiles(L, tile):
    """Number of tiles covering L rows (the last one may be ragged)."""
    return -(-int(L) // int(tile))


def n_groups(nkt, g):
    """Number of key-tile groups of g tiles covering nkt key tiles (reading (e))."""
    return -(-int(nkt) // int(g))


def mask_words(max_lk, tile_n, g):
    """32-bit words per query-tile row of the bitmask: ceil(n_groups / 32)."""
    return max(1, -(-n_groups(n_tiles(max_lk, tile_n), g) // 32))


def tile_table(seqs, tile, side):
    """All tiles of one side in global order.

    Returns a list of (b, I, row_start, rows, I_glob): tile I of sequence b
    covers global rows row_start .. row_start + rows - 1; I_glob numbers the
    tiles of all sequences in order, each sequence starting a new tile.
    ``side`` is "q" (uses q_start/Lq) or "k" (uses k_start/Lk).
    """
    out = []
    glob = 0
    for b, (qs, lq, ks, lk) in enumerate(seqs):
        start, length = (qs, lq) if side == "q" else (ks, lk)
        for i in range(n_tiles(length, tile)):
            r0 = i * tile
            out.append((b, i, start + r0, min(tile, length - r0), glob))
            glob += 1
    return out


def visible(i, j, Lq, Lk, causal):
    """Key j is visible to query i (reading (f), bottom-right causal)."""
    i = np.asarray(i)
    j = np.asarray(j)
    ok = j < Lk
    if causal:
        ok = ok & (j <= i + (Lk - Lq))
    return ok


def last_visible_key(i_last, Lq, Lk, causal):
    """Largest key index visible to query row i_last (-1 if none)."""
    if Lk <= 0:
        return -1
    if not causal:
        return Lk - 1
    return min(Lk - 1, i_last + Lk - Lq)


# --------------------------------------------------------------------------
# quantiser (reading (a))
# --------------------------------------------------------------------------

def quantize_tiles(x16, seqs, tile, side):
    """Per-(head, tile) symmetric absmax/127 quantisation.

    x16: float16 [T, H, d].  For every tile of ``tile_table(seqs, tile, side)``
    and every head h: amax = max |x| over the tile's rows x d (exact: fp16 ->
    fp32 is exact); s = fl32(amax / 127) by IEEE fp32 division; codes =
    clamp(rne(fl32(x / s)), -127, 127), x and s in fp32; amax == 0 gives s = 0
    and codes 0.  Returns (codes int8 [T, H, d], scales float32 [n_tiles, H]),
    tiles in the global order of ``tile_table``.
    Rows outside every tile keep code 0.
    """
    x16 = np.asarray(x16, dtype=np.float16)
    T, H, d = x16.shape
    tiles = tile_table(seqs, tile, side)
    codes = np.zeros((T, H, d), dtype=np.int8)
    scales = np.zeros((len(tiles), H), dtype=np.float32)
    x32 = x16.astype(np.float32)
    for (_b, _i, r0, rows, ig) in tiles:
        for h in range(H):
            blk = x32[r0:r0 + rows, h, :]
            amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
            s = np.float32(amax / np.float32(127.0))
            scales[ig, h] = s
            if s == 0:
                continue
            q = np.rint(blk / s)                      # fp32 division, then RNE
            codes[r0:r0 + rows, h, :] = np.clip(q, -127, 127).astype(np.int8)
    return codes, scales


# --------------------------------------------------------------------------
# FP8 E4M3 (reading (p))
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Values of FP8 E4M3 codes (uint8): bit 7 sign, bits 6..3 exponent
    (bias 7), bits 2..0 mantissa; exponent 0 is subnormal, m/8 * 2^-6;
    exponent 15 with mantissa 7 is NaN (the format has no infinities, so
    exponent 15 with mantissa 0..6 are finite values up to 448)."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


_E4M3_MAGS = None


def e4m3_encode(x):
    """E4M3 codes (uint8) of fp32 values: the nearest finite E4M3 value, ties
    to the code with an even mantissa, magnitudes beyond 448 saturating to 448
    ("satfinite"); the sign bit is the sign of x (so a negative value that
    rounds to zero gives the code of -0)."""
    global _E4M3_MAGS
    if _E4M3_MAGS is None:
        _E4M3_MAGS = e4m3_decode(np.arange(0, 0x7F))       # codes 0x00..0x7E, ascending magnitudes
    mags = _E4M3_MAGS
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, len(mags) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - mags[lo], mags[hi] - a
    take_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.int64)
    code = np.where(np.signbit(x), code | 0x80, code)
    return code.astype(np.uint8)


def quantize_tiles_fp8(x16, seqs, tile, side):
    """Per-(head, tile) FP8 E4M3 quantisation, reading (p): amax = max |x|
    over the tile's rows x d; s = fl32(amax / 448); codes = e4m3_encode(
    fl32(x / s)); amax == 0 gives s = 0 and codes 0.  Returns (codes uint8
    [T, H, d], scales float32 [n_tiles, H]) in the tile order of
    ``tile_table``; rows outside every tile keep code 0."""
    x16 = np.asarray(x16, dtype=np.float16)
    T, H, d = x16.shape
    tiles = tile_table(seqs, tile, side)
    codes = np.zeros((T, H, d), dtype=np.uint8)
    scales = np.zeros((len(tiles), H), dtype=np.float32)
    x32 = x16.astype(np.float32)
    for (_b, _i, r0, rows, ig) in tiles:
        for h in range(H):
            blk = x32[r0:r0 + rows, h, :]
            amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
            s = np.float32(amax / np.float32(E4M3_MAX))
            scales[ig, h] = s
            if s == 0:
                continue
            codes[r0:r0 + rows, h, :] = e4m3_encode(blk / s)   # fp32 division
    return codes, scales


def dequant_cache(codes, scale16):
    """FP16 view of an INT8 cache: fp16_rn(fl32(code) * fl32(scale)).

    codes int8 [T, H, d]; scale16 float16 [T, H] (one scale per token and
    head).  The fp32 product is exact (8 + 11 significant bits), so the only
    rounding is the final one to fp16.
    """
    c = np.asarray(codes, dtype=np.int8).astype(np.float32)
    s = np.asarray(scale16, dtype=np.float16).astype(np.float32)
    return (c * s[..., None]).astype(np.float16)


# --------------------------------------------------------------------------
# routing bitmask (reading (m))
# --------------------------------------------------------------------------

def splitmix64(x):
    """SplitMix64 output function (Steele, Lea and Flood, OOPSLA 2014):
    add the golden-ratio increment, then two xor-shift-multiply rounds and a
    final xor-shift.  Works on Python ints or numpy uint64 arrays (mod 2^64).
    """
    if isinstance(x, np.ndarray):
        with np.errstate(over="ignore"):
            z = x.astype(np.uint64) + np.uint64(SPLITMIX_GAMMA)
            z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
            z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
            return z ^ (z >> np.uint64(31))
    z = (int(x) + SPLITMIX_GAMMA) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _legal_groups(qtile, seqs, tile_m, tile_n, g, causal):
    """(number of legal groups, index of the diagonal group) for one q tile."""
    b, i, _r0, rows, _ig = qtile
    _qs, lq, _ks, lk = seqs[b]
    jmax = last_visible_key(i * tile_m + rows - 1, lq, lk, causal)
    if jmax < 0:
        return 0, -1
    nj = jmax // tile_n + 1
    return (nj - 1) // g + 1, (nj - 1) // g


def build_mask(Hq, seqs, tile_m, tile_n, g, causal, p, seed,
               force_diag=False, force_sink=False, words=None):
    """Seeded Bernoulli routing bitmask, uint32 [Hq, n_qtiles, W].

    Word (h, I_glob, G // 32), bit G % 32 is 1 (INT8) iff group G is legal
    for query tile I_glob, is not forced, and u < p, where
      u = (splitmix64(seed XOR (h * 2^40 + I_glob * 2^20 + G)) >> 11) * 2^-53.
    Forced groups (diagonal when force_diag, group 0 when force_sink) and
    illegal groups are 0.  W defaults to mask_words(max Lk, tile_n, g).
    """
    qt = tile_table(seqs, tile_m, "q")
    if words is None:
        words = mask_words(max([s[3] for s in seqs] + [1]), tile_n, g)
    out = np.zeros((Hq, len(qt), words), dtype=np.uint32)
    seed = int(seed) & _M64
    for t in qt:
        ig = t[4]
        ng, gdiag = _legal_groups(t, seqs, tile_m, tile_n, g, causal)
        if ng == 0:
            continue
        G = np.arange(ng, dtype=np.uint64)
        for h in range(Hq):
            key = (np.uint64(h) << np.uint64(40)) + (np.uint64(ig) << np.uint64(20)) + G
            u = (splitmix64(np.uint64(seed) ^ key) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
            bit = u < p
            if force_sink:
                bit[0] = False
            if force_diag:
                bit[gdiag] = False
            for gi in np.nonzero(bit)[0]:
                out[h, ig, gi // 32] |= np.uint32(1 << (int(gi) % 32))
    return out


def build_mask_scale_policy(Hq, Hkv, seqs, tile_m, tile_n, g, causal, q_scales, k_scales, tau,
                            force_diag=False, force_sink=False, words=None, k_token_scales=None):
    """Content-driven routing bitmask from the tile quantisation scales,
    uint32 [Hq, n_qtiles, W] in the layout of ``build_mask``.

    TileMix (Lattice paper page, abstract) adjusts precision during inference
    and claims a controllable accuracy-efficiency frontier, but gives no
    policy.  Plainest content signal: with symmetric absmax/127 codes every
    element's rounding error is at most half a step, so the INT8 score of a
    tile pair differs from the fp16 one by at most
        d * s_q[I] * s_k[J] * (127 + 1/4)
    (|q| <= 127 s_q, |k| <= 127 s_k).  A group is routed INT8 when this bound,
    taken over the group's key tiles that query tile I sees, is at most a
    threshold: with mk = max of s_k over key tiles J in
    [G*g, min((G+1)*g, nj)) (nj = key tiles visible to I; kv head
    h // (Hq/Hkv)), bit = fl32(s_q[I, h] * mk) <= tau (fp32).  Legality and
    forcing are those of ``build_mask``.  tau = +inf routes every eligible
    group INT8; tau < 0 none.
    q_scales: fp32 [n_qtiles, Hq]; k_scales: fp32 [n_ktiles, Hkv], global
    tile order of ``tile_table``.  The sequences may have their own key
    offsets (``seq_table`` with ``cu_seqlens_k``): key tiles, legality and
    causality then follow each sequence's (Lq, Lk).

    k_token_scales (instead of k_scales): fp16 [Tk, Hkv], one scale per key
    token, as an INT8 cache carries.  The FP16 route then reads the fp16 view
    k^ = fp16(c_k * s_k) and the INT8 route s_q * s_k * (c_q . c_k), so per
    score the two differ by at most about d * s_q * s_k * (127/2 + 127^2 / 2^11)
    (half a step of Q rounding times |c_k| <= 127, plus the fp16 rounding of
    the dequantised key), again proportional to s_q * s_k.  mk is then the
    largest fp32 value of s_k over the key tokens of the group's visible key
    tiles: rows [G*g*tile_n, min(min((G+1)*g, nj)*tile_n, Lk)) of the
    sequence's keys.
    """
    if (k_scales is None) == (k_token_scales is None):
        raise ValueError("give k_scales (per key tile) or k_token_scales (per key token)")
    qt = tile_table(seqs, tile_m, "q")
    kt = tile_table(seqs, tile_n, "k")
    kbase = {}
    for (b, i, _r0, _rows, ig) in kt:
        if i == 0:
            kbase[b] = ig
    if words is None:
        words = mask_words(max([s[3] for s in seqs] + [1]), tile_n, g)
    q_scales = np.asarray(q_scales, dtype=np.float32)
    if k_scales is not None:
        k_scales = np.asarray(k_scales, dtype=np.float32)
    else:
        k_tok = np.asarray(k_token_scales, dtype=np.float16).astype(np.float32)
    tau = np.float32(tau)
    grp = Hq // Hkv
    out = np.zeros((Hq, len(qt), words), dtype=np.uint32)
    for t in qt:
        b, _i, _r0, _rows, ig = t
        ng, gdiag = _legal_groups(t, seqs, tile_m, tile_n, g, causal)
        if ng == 0:
            continue
        jmax = last_visible_key(t[1] * tile_m + t[3] - 1, seqs[b][1], seqs[b][3], causal)
        nj = jmax // tile_n + 1
        for h in range(Hq):
            hk = h // grp
            sq = q_scales[ig, h]
            for G in range(ng):
                if (force_sink and G == 0) or (force_diag and G == gdiag):
                    continue
                j1 = min((G + 1) * g, nj)
                if k_scales is not None:
                    mk = max(k_scales[kbase[b] + j, hk] for j in range(G * g, j1))
                else:
                    k0 = seqs[b][2]
                    r_end = min(j1 * tile_n, seqs[b][3])
                    mk = max(k_tok[k0 + r, hk] for r in range(G * g * tile_n, r_end))
                if np.float32(sq * mk) <= tau:
                    out[h, ig, G // 32] |= np.uint32(1 << (G % 32))
    return out


def mask_bit(mask, h, ig, G):
    """Routing bit of group G of query tile ig for head h (head stride 0 when
    the mask has a single head plane)."""
    hh = 0 if mask.shape[0] == 1 else h
    return (int(mask[hh, ig, G // 32]) >> (G % 32)) & 1


def _group_bits(mask, h, ig, ng):
    """Bits of groups 0 .. ng-1 of query tile ig, head h, as a bool array."""
    hh = 0 if mask.shape[0] == 1 else h
    G = np.arange(ng)
    words = mask[hh, ig, G // 32].astype(np.uint64)
    return ((words >> (G % 32).astype(np.uint64)) & np.uint64(1)).astype(bool)


def route_stats(mask, seqs, Hq, tile_m, tile_n, g, causal):
    """(N_vis, E8): visible query-key pairs over all heads and sequences, and
    those lying in INT8-routed tiles.  The realised INT8 fraction is E8/N_vis."""
    n_vis = 0
    e8 = 0
    for t in tile_table(seqs, tile_m, "q"):
        b, i, _r0, rows, ig = t
        _qs, lq, _ks, lk = seqs[b]
        ii = i * tile_m + np.arange(rows)
        jlim = np.minimum(lk - 1, ii + (lk - lq)) if causal else np.full(rows, lk - 1)
        cnt_row = np.maximum(jlim + 1, 0)
        tile_vis = int(cnt_row.sum())
        n_vis += Hq * tile_vis
        if mask is None or tile_vis == 0:
            continue
        nj = int(jlim.max()) // tile_n + 1
        per_tile = np.array([int(np.clip(jlim - J * tile_n + 1, 0, tile_n).sum()) for J in range(nj)])
        for h in range(Hq):
            bits = _group_bits(mask, h, ig, n_groups(nj, g))
            e8 += int(per_tile[bits[np.arange(nj) // g]].sum())
    return n_vis, e8


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def attention(q, k=None, v=None, *, cu_seqlens=None, causal=False,
              tile_m=128, tile_n=128, g=1, mask=None,
              q_quant=None, k_quant=None, kv_cache=None, rows=None, cu_seqlens_k=None,
              mask_fp8=None, qf8_quant=None, kf8_quant=None):
    """Tile-routed softmax attention in fp64.  Returns float64 [Tq, Hq, d].

    q: float16 [Tq, Hq, d]; k, v: float16 [Tk, Hkv, d] (or None with an INT8
    cache).  mask: uint32 [Hq or 1, n_qtiles, W] or None (all FP16).
    q_quant = (codes, scales[n_qtiles, Hq]) and k_quant = (codes,
    scales[n_ktiles, Hkv]) are the tile-quantised operands of the INT8 route.
    kv_cache = (k_codes, k_scale16[Tk, Hkv], v_codes, v_scale16) replaces k, v:
    the FP16 route and P.V use the fp16 view (dequant_cache), the INT8 route
    uses k_codes with the per-token scale of each key.
    rows: optional iterable of global query rows to evaluate (others are NaN).
    cu_seqlens_k: key offsets per sequence when they differ from cu_seqlens
    (prefix-cached prefill); reading (j).
    mask_fp8 (reading (p)): a second bit plane in the layout of ``mask``; a
    legal group whose INT8 bit is clear and FP8 bit is set takes
    S_ij = sigma * s_q * s_k * (dot product of the E4M3-decoded codes), with
    qf8_quant = (codes, scales[n_qtiles, Hq]) and kf8_quant = (codes,
    scales[n_ktiles, Hkv]) from quantize_tiles_fp8 (fp16 K only).

    For each sequence, query head h (KV head hk = h // (Hq/Hkv)) and visible
    pair (i, j) in query tile I (global I_glob), key tile J, group G = J // g:
      FP16 route: S_ij = sigma * sum_t q_it k_jt   (fp16 values, fp64 sums)
      INT8 route: S_ij = sigma * s_q[I_glob, h] * s_k * sum_t cq_it ck_jt
    with s_k = k tile scale (or the cache scale of key j); the integer sum is
    exact in fp64.  O_i = sum_j softmax_j(S_i.) V_j over visible j; a row with
    no visible key gives 0.
    """
    q = np.asarray(q, dtype=np.float16)
    Tq, Hq, d = q.shape
    if kv_cache is not None:
        kc, ks16, vc, vs16 = kv_cache
        k16 = dequant_cache(kc, ks16)
        v16 = dequant_cache(vc, vs16)
    else:
        k16 = np.asarray(k, dtype=np.float16)
        v16 = np.asarray(v, dtype=np.float16)
    Tk, Hkv, _ = k16.shape
    assert Hq % Hkv == 0
    grp = Hq // Hkv
    sigma = 1.0 / math.sqrt(d)
    seqs = seq_table(Tq, Tk, cu_seqlens, cu_seqlens_k)
    qtiles = tile_table(seqs, tile_m, "q")
    kt_off = []
    acc = 0
    for (_qs, _lq, _ks, lk) in seqs:
        kt_off.append(acc)
        acc += n_tiles(lk, tile_n)
    want = None
    if rows is not None:
        want = np.zeros(Tq, dtype=bool)
        want[np.asarray(list(rows), dtype=np.int64)] = True

    out = np.full((Tq, Hq, d), np.nan if rows is not None else 0.0, dtype=np.float64)
    kf = k16.astype(np.float64)
    vf = v16.astype(np.float64)
    if mask_fp8 is not None:
        if kv_cache is not None:
            raise ValueError("the FP8 route takes tile-quantised fp16 K, not an INT8 cache")
        qf8_val = e4m3_decode(qf8_quant[0])
        kf8_val = e4m3_decode(kf8_quant[0])
        qf8_scales = np.asarray(qf8_quant[1], dtype=np.float32)
        kf8_scales = np.asarray(kf8_quant[1], dtype=np.float32)
    if mask is not None:
        q_codes = np.asarray(q_quant[0])
        q_scales = np.asarray(q_quant[1], dtype=np.float32)
        if kv_cache is not None:
            k_codes = np.asarray(kv_cache[0]).astype(np.float64)
            k_tok_scale = np.asarray(kv_cache[1], dtype=np.float16).astype(np.float64)
        else:
            k_codes = np.asarray(k_quant[0]).astype(np.float64)
            k_tile_scale = np.asarray(k_quant[1], dtype=np.float32)

    for (b, I, r0, nrows, ig) in qtiles:
        qs, lq, ks, lk = seqs[b]
        sel = np.arange(nrows)
        if want is not None:
            sel = sel[want[r0:r0 + nrows]]
            if sel.size == 0:
                continue
        ii = I * tile_m + sel                        # row index within the sequence
        jj = np.arange(lk)
        vis = visible(ii[:, None], jj[None, :], lq, lk, causal)
        for h in range(Hq):
            hk = h // grp
            Kb = kf[ks:ks + lk, hk, :]
            Vb = vf[ks:ks + lk, hk, :]
            Qr = q[r0 + sel, h, :].astype(np.float64)
            S = sigma * (Qr @ Kb.T)
            route8 = np.zeros(lk, dtype=bool)
            if mask is not None:
                route8 = _group_bits(mask, h, ig, n_groups(n_tiles(lk, tile_n), g))[(jj // tile_n) // g]
                if route8.any():
                    acc8 = q_codes[r0 + sel, h, :].astype(np.float64) @ k_codes[ks:ks + lk, hk, :].T
                    if kv_cache is not None:
                        col_scale = k_tok_scale[ks:ks + lk, hk]
                    else:
                        col_scale = k_tile_scale[kt_off[b] + jj // tile_n, hk].astype(np.float64)
                    S8 = sigma * float(q_scales[ig, h]) * acc8 * col_scale[None, :]
                    S = np.where(route8[None, :], S8, S)
            if mask_fp8 is not None:
                routef8 = ~route8 & _group_bits(mask_fp8, h, ig, n_groups(n_tiles(lk, tile_n), g))[(jj // tile_n) // g]
                if routef8.any():
                    accf8 = qf8_val[r0 + sel, h, :] @ kf8_val[ks:ks + lk, hk, :].T    # exact in fp64
                    colf8 = kf8_scales[kt_off[b] + jj // tile_n, hk].astype(np.float64)
                    Sf8 = sigma * float(qf8_scales[ig, h]) * accf8 * colf8[None, :]
                    S = np.where(routef8[None, :], Sf8, S)
            S = np.where(vis, S, -np.inf)
            has = vis.any(axis=1)
            m = np.where(has, S.max(axis=1, initial=-np.inf), 0.0)
            P = np.where(vis, np.exp(S - m[:, None]), 0.0)
            lsum = P.sum(axis=1)
            O = P @ Vb
            O = np.where(has[:, None], O / np.where(has, lsum, 1.0)[:, None], 0.0)
            out[r0 + sel, h, :] = O
    return out


def attention_rows(q, k=None, v=None, rows=(), **kw):
    """``attention`` evaluated on the given global query rows only."""
    return attention(q, k, v, rows=rows, **kw)
