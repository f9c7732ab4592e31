"""Pins of the oracle's routing bitmask: one bit per (query tile, group of g
key tiles), 1 = INT8, drawn by a counter-based hash.

Source: TileMix (Lattice paper page), abstract -- routing decisions packed
into a bitmask, one bit for several neighbouring key tiles, every legal tile
group computed.  The Bernoulli draw, the forced diagonal/sink groups and the word
layout are the readings stated in the oracle's module docstring.
"""

import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_vectors():
    rows = [l.split() for l in open(os.path.join(GOLD, "splitmix64_vectors.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) >= 2
    for n, hx in rows:
        x = (int(n) * oracle.SPLITMIX_GAMMA) % (1 << 64)
        assert oracle.splitmix64(x) == int(hx, 16)
        # numpy path agrees with the integer path
        assert int(oracle.splitmix64(np.array([x], dtype=np.uint64))[0]) == int(hx, 16)


def test_mask_words_formula():
    assert oracle.mask_words(16384, 128, 4) == 1          # 128 tiles / 4 = 32 groups
    assert oracle.mask_words(16385, 128, 4) == 2          # 129 tiles -> 33 groups
    assert oracle.mask_words(65536, 128, 8) == 2          # 512 / 8 = 64 groups
    assert oracle.mask_words(256, 64, 1) == 1
    assert oracle.mask_words(1, 128, 1) == 1


def _eligible(seqs, Hq, tm, tn, g, causal, fd, fs):
    """Brute-force count of groups that may carry a 1: legal and not forced."""
    n = 0
    for t in oracle.tile_table(seqs, tm, "q"):
        b, i, r0, rows, ig = t
        _qs, lq, _ks, lk = seqs[b]
        legal = set()
        for r in range(rows):
            for j in range(lk):
                if oracle.visible(i * tm + r, j, lq, lk, causal):
                    legal.add((j // tn) // g)
        if not legal:
            continue
        last_tile = max(j // tn for r in range(rows) for j in range(lk)
                        if oracle.visible(i * tm + r, j, lq, lk, causal))
        for G in legal:
            if fd and G == last_tile // g:
                continue
            if fs and G == 0:
                continue
            n += Hq
    return n


CASES = [
    # (Tq, Tk, cu, Hq, tm, tn, g, causal, fd, fs)
    (300, 300, None, 2, 64, 64, 1, True, True, True),
    (300, 300, None, 2, 64, 64, 2, False, False, False),
    (100, 400, None, 3, 32, 64, 3, True, True, False),
    (400, 100, None, 1, 64, 32, 1, True, False, True),     # Lq > Lk: empty q tiles
    (0, 0, [0, 130, 130, 390], 2, 64, 64, 2, True, True, True),
]


@pytest.mark.parametrize("case", CASES)
def test_p1_sets_exactly_the_eligible_groups(case):
    Tq, Tk, cu, Hq, tm, tn, g, causal, fd, fs = case
    if cu is not None:
        Tq = Tk = cu[-1]
    seqs = oracle.seq_table(Tq, Tk, cu)
    m1 = oracle.build_mask(Hq, seqs, tm, tn, g, causal, 1.0, 123, fd, fs)
    m0 = oracle.build_mask(Hq, seqs, tm, tn, g, causal, 0.0, 123, fd, fs)
    assert not m0.any()
    ones = int(np.unpackbits(m1.view(np.uint8)).sum())
    assert ones == _eligible(seqs, Hq, tm, tn, g, causal, fd, fs)


def test_illegal_and_forced_groups_are_zero():
    L, tm, tn, g = 1024, 64, 64, 2
    seqs = oracle.seq_table(L, L)
    m = oracle.build_mask(4, seqs, tm, tn, g, True, 1.0, 5, True, True)
    nqt = L // tm
    for h in range(4):
        for I in range(nqt):
            diag = (I * tm + tm - 1) // tn // g
            for G in range(oracle.n_groups(L // tn, g)):
                bit = oracle.mask_bit(m, h, I, G)
                if G > diag or G == diag or G == 0:
                    assert bit == 0
                else:
                    assert bit == 1


@pytest.mark.parametrize("p", [0.25, 0.5, 0.75])
def test_realised_fraction_is_binomial(p):
    L = 8192
    seqs = oracle.seq_table(L, L)
    m = oracle.build_mask(8, seqs, 128, 128, 1, False, p, 99)
    n = 8 * (L // 128) * (L // 128)
    ones = int(np.unpackbits(m.view(np.uint8)).sum())
    sd = (n * p * (1 - p)) ** 0.5
    assert abs(ones - n * p) < 5 * sd


def test_seeded_and_deterministic():
    seqs = oracle.seq_table(2048, 2048)
    a = oracle.build_mask(2, seqs, 128, 128, 1, True, 0.5, 1)
    b = oracle.build_mask(2, seqs, 128, 128, 1, True, 0.5, 1)
    c = oracle.build_mask(2, seqs, 128, 128, 1, True, 0.5, 2)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)


def test_hash_key_layout():
    # bit (h, I, G) is decided by splitmix64(seed ^ (h<<40 | I<<20 | G)) >> 11 < p * 2^53
    seqs = oracle.seq_table(1024, 1024)
    seed = 0xDEADBEEF12345
    m = oracle.build_mask(3, seqs, 128, 128, 1, False, 0.5, seed)
    for h in range(3):
        for I in range(8):
            for G in range(8):
                u = oracle.splitmix64(seed ^ ((h << 40) + (I << 20) + G)) >> 11
                assert oracle.mask_bit(m, h, I, G) == int(u < (1 << 52))


def test_route_stats_counts_pairs():
    # causal square, tiles 2: N_vis = L(L+1)/2 per head
    L, Hq = 10, 3
    seqs = oracle.seq_table(L, L)
    m = oracle.build_mask(Hq, seqs, 2, 2, 1, True, 1.0, 0)
    n_vis, e8 = oracle.route_stats(m, seqs, Hq, 2, 2, 1, True)
    assert n_vis == Hq * L * (L + 1) // 2
    # every legal tile is INT8 with p = 1 and nothing forced
    assert e8 == n_vis
    n_vis2, e82 = oracle.route_stats(None, seqs, Hq, 2, 2, 1, True)
    assert n_vis2 == n_vis and e82 == 0
    # bottom-right with Lq > Lk: the first Lq - Lk rows see nothing
    seqs = oracle.seq_table(12, 5)
    n_vis, _ = oracle.route_stats(None, seqs, 1, 4, 4, 1, True)
    assert n_vis == sum(max(0, min(5, i + 5 - 12 + 1)) for i in range(12))


# ------------------------------------------------------------------ scale policy
# Content-driven routing (the frontier item): a group is INT8 when
# s_q * max s_k over its key tiles is at most tau.  Pins: the extremes reduce
# to the Bernoulli builder's p = 1 / p = 0 masks, the mask is monotone in tau,
# a key tile made an outlier by construction is exactly the one kept FP16, and
# the error bound the policy thresholds holds for INT8 scores.

def _policy_case(lens, causal, tile, g, hq=4, hkv=2, d=16, seed=3, outlier=None):
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    seqs = oracle.seq_table(cu[-1], cu[-1], cu)
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((cu[-1], hq, d)).astype(np.float16)
    k = rng.standard_normal((cu[-1], hkv, d)).astype(np.float16)
    if outlier is not None:
        rows, val = outlier
        k[rows, :, 0] = np.float16(val)
    _, qs = oracle.quantize_tiles(q, seqs, tile, "q")
    _, ks = oracle.quantize_tiles(k, seqs, tile, "k")
    return seqs, qs, ks


@pytest.mark.parametrize("lens,causal,g,fd,fs", [
    ([300], True, 1, False, False), ([300], False, 2, True, True), ([70, 200, 129], True, 3, True, False),
])
def test_scale_policy_extremes_equal_bernoulli_p1_and_p0(lens, causal, g, fd, fs):
    seqs, qs, ks = _policy_case(lens, causal, 32, g)
    kw = dict(force_diag=fd, force_sink=fs)
    all_on = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, g, causal, qs, ks, np.inf, **kw)
    assert np.array_equal(all_on, oracle.build_mask(4, seqs, 32, 32, g, causal, 1.0, 7, **kw))
    none = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, g, causal, qs, ks, -1.0, **kw)
    assert not none.any()


def test_scale_policy_monotone_in_tau():
    seqs, qs, ks = _policy_case([257, 96], True, 32, 2)
    prods = np.sort(np.outer(qs.ravel(), ks.ravel()).ravel())
    prev = None
    for tau in np.quantile(prods, [0.0, 0.1, 0.3, 0.5, 0.7, 0.9, 1.0]):
        m = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, 2, True, qs, ks, tau)
        if prev is not None:
            assert np.array_equal(prev & m, prev)       # bits only ever turn on
        prev = m


def test_scale_policy_keeps_the_outlier_key_tile_fp16():
    # one sequence of 8 key tiles of 32 rows; key tile 5 carries a value 100x
    # the others in channel 0 of every kv head, so its scale is ~25x larger
    tile, g = 32, 2
    seqs, qs, ks = _policy_case([256], False, tile, g, outlier=(slice(5 * tile, 6 * tile), 400.0))
    normal = np.float32(qs.max()) * np.float32(np.delete(ks, 5, axis=0).max())
    tau = np.float32(normal * 1.01)
    m = oracle.build_mask_scale_policy(4, 2, seqs, tile, tile, g, False, qs, ks, tau)
    outlier_group = 5 // g
    for h in range(4):
        for ig in range(8):
            bits = [oracle.mask_bit(m, h, ig, G) for G in range(4)]
            assert bits == [0 if G == outlier_group else 1 for G in range(4)], (h, ig, bits)


def test_int8_score_error_within_the_policy_bound():
    # |s_q s_k (c_q . c_k) - q . k| <= d * s_q * s_k * (127 + 1/4), per score
    rng = np.random.default_rng(11)
    d = 64
    for scale_q, scale_k in ((1.0, 1.0), (20.0, 0.05), (1e-3, 300.0)):
        q = (rng.standard_normal((32, 1, d)) * scale_q).astype(np.float16)
        k = (rng.standard_normal((32, 1, d)) * scale_k).astype(np.float16)
        q[3, 0, :4] *= np.float16(20)                                # outlier channels
        seqs = oracle.seq_table(32, 32)
        qc, qs = oracle.quantize_tiles(q, seqs, 32, "q")
        kc, ks = oracle.quantize_tiles(k, seqs, 32, "k")
        s8 = float(qs[0, 0]) * float(ks[0, 0]) * (qc[:, 0].astype(np.float64) @ kc[:, 0].astype(np.float64).T)
        s16 = q[:, 0].astype(np.float64) @ k[:, 0].astype(np.float64).T
        bound = d * float(qs[0, 0]) * float(ks[0, 0]) * (127 + 0.25)
        assert np.abs(s8 - s16).max() <= bound


# -------------------------------------------- scale policy: key offsets, INT8 cache
# The policy with separate key offsets (prefix-cached prefill) and with one key
# scale per token (INT8 cache).  Pins: brute force over visible pairs, the
# extremes, monotonicity, reduction to the tile-scale policy, an outlier token
# placed by construction, and the cache score-error bound the policy thresholds.

def _prefix_case(lens_q, lens_k, hq=4, hkv=2, d=16, seed=5, tile=32):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).tolist()
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).tolist()
    seqs = oracle.seq_table(cu_q[-1], cu_k[-1], cu_q, cu_k)
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((cu_q[-1], hq, d)).astype(np.float16)
    _, qs = oracle.quantize_tiles(q, seqs, tile, "q")
    # per-token cache scales: fp16, spread over two decades
    ktok = (10.0 ** rng.uniform(-3, -1, size=(cu_k[-1], hkv))).astype(np.float16)
    return seqs, qs, ktok


def _brute_policy(Hq, Hkv, seqs, tile_m, tile_n, g, causal, qs, ktok, tau, words):
    """Bits from the visible pairs themselves: group G of query tile I counts
    the key tiles of G holding a key that some row of I sees; mk is the
    largest token scale over all tokens of those tiles."""
    out = np.zeros((Hq, len(oracle.tile_table(seqs, tile_m, "q")), words), dtype=np.uint32)
    for (b, I, _r0, rows, ig) in oracle.tile_table(seqs, tile_m, "q"):
        _qs0, lq, k0, lk = seqs[b]
        ii = I * tile_m + np.arange(rows)
        for J in range(oracle.n_tiles(lk, tile_n)):
            jj = np.arange(J * tile_n, min((J + 1) * tile_n, lk))
            if not oracle.visible(ii[:, None], jj[None, :], lq, lk, causal).any():
                continue
            G = J // g
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                # max over every visible tile of the group (recomputed per tile)
                tiles = [Jx for Jx in range(G * g, min((G + 1) * g, oracle.n_tiles(lk, tile_n)))
                         if oracle.visible(ii[:, None],
                                           np.arange(Jx * tile_n, min((Jx + 1) * tile_n, lk))[None, :],
                                           lq, lk, causal).any()]
                mk = max(np.float32(ktok[k0 + r, hk]) for Jx in tiles
                         for r in range(Jx * tile_n, min((Jx + 1) * tile_n, lk)))
                if np.float32(np.float32(qs[ig, h]) * mk) <= np.float32(tau):
                    out[h, ig, G // 32] |= np.uint32(1 << (G % 32))
    return out


@pytest.mark.parametrize("lens_q,lens_k,causal,g", [
    ([40], [130], True, 1), ([40, 65, 1], [130, 65, 97], True, 2), ([33, 70], [20, 150], False, 3),
])
def test_token_policy_matches_brute_force_over_visible_pairs(lens_q, lens_k, causal, g):
    seqs, qs, ktok = _prefix_case(lens_q, lens_k)
    W = oracle.mask_words(max(lens_k), 32, g)
    full = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, g, causal, qs, None, np.inf, words=W,
                                          k_token_scales=ktok)
    partial = 0
    for tau in np.quantile(np.outer(qs.ravel(), ktok.astype(np.float32).ravel()), [0.9, 0.97, 0.995]):
        m = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, g, causal, qs, None, tau, words=W,
                                           k_token_scales=ktok)
        assert np.array_equal(m, _brute_policy(4, 2, seqs, 32, 32, g, causal, qs, ktok, tau, W))
        partial += int(m.any() and not np.array_equal(m, full))
    assert partial >= 1          # at least one threshold splits the groups


@pytest.mark.parametrize("fd,fs", [(False, False), (True, True)])
def test_key_offset_policy_extremes_equal_bernoulli_p1_and_p0(fd, fs):
    seqs, qs, ktok = _prefix_case([40, 65, 1], [130, 65, 97])
    kw = dict(force_diag=fd, force_sink=fs)
    on = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, 2, True, qs, None, np.inf, k_token_scales=ktok, **kw)
    assert np.array_equal(on, oracle.build_mask(4, seqs, 32, 32, 2, True, 1.0, 9, **kw))
    off = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, 2, True, qs, None, -1.0, k_token_scales=ktok, **kw)
    assert not off.any()


def test_token_policy_monotone_in_tau():
    seqs, qs, ktok = _prefix_case([70, 33], [200, 90])
    prods = np.sort(np.outer(qs.ravel(), ktok.astype(np.float32).ravel()).ravel())
    prev = None
    for tau in np.quantile(prods, [0.0, 0.2, 0.4, 0.6, 0.8, 1.0]):
        m = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, 1, True, qs, None, tau, k_token_scales=ktok)
        if prev is not None:
            assert np.array_equal(prev & m, prev)
        prev = m


def test_token_policy_reduces_to_tile_policy_for_tile_constant_scales():
    # token scales constant within each key tile: the per-token policy must
    # give the per-tile policy's bits with those tile scales
    seqs, qs, ktok = _prefix_case([40, 65, 1], [130, 65, 97])
    kt = oracle.tile_table(seqs, 32, "k")
    tile_sc = np.zeros((len(kt), 2), dtype=np.float32)
    for (b, _i, r0, rows, ig) in kt:
        ktok[r0:r0 + rows] = ktok[r0]
        tile_sc[ig] = ktok[r0].astype(np.float32)
    for tau in np.quantile(np.outer(qs.ravel(), tile_sc.ravel()), [0.25, 0.5, 0.75]):
        a = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, 2, True, qs, None, tau, k_token_scales=ktok)
        b = oracle.build_mask_scale_policy(4, 2, seqs, 32, 32, 2, True, qs, tile_sc, tau)
        assert np.array_equal(a, b)


def test_token_policy_keeps_only_the_outlier_tokens_group_fp16():
    # one sequence, 64 queries after a 192-key prefix (Lk = 256, causal,
    # bottom-right); every token scale is 1e-3 except key 5*32+7 = 167 at 1.0
    tile, g = 32, 2
    lq, lk = 64, 256
    seqs = oracle.seq_table(lq, lk)
    qs = np.full((2, 4), 0.01, dtype=np.float32)
    ktok = np.full((lk, 2), 1e-3, dtype=np.float16)
    ktok[5 * tile + 7, :] = 1.0
    tau = np.float32(0.01) * np.float32(np.float16(1e-3)) * np.float32(2)
    m = oracle.build_mask_scale_policy(4, 2, seqs, tile, tile, g, True, qs, None, tau, k_token_scales=ktok)
    for h in range(4):
        for I in range(2):
            ng = (lk - lq + (I + 1) * tile - 1) // tile // g + 1     # groups query tile I sees
            bits = [oracle.mask_bit(m, h, I, G) for G in range(ng)]
            assert bits == [0 if G == 5 // g else 1 for G in range(ng)], (h, I, bits)


def test_cache_int8_score_error_within_the_token_policy_bound():
    # |s_q s_k (c_q . c_k) - q . fp16(c_k s_k)| <= d s_q s_k (127/2 + 127^2 / 2^11), per score
    rng = np.random.default_rng(13)
    d = 64
    for scale_q in (1.0, 30.0, 2e-3):
        q = (rng.standard_normal((32, 1, d)) * scale_q).astype(np.float16)
        q[5, 0, :3] *= np.float16(16)
        seqs = oracle.seq_table(32, 32)
        qc, qsc = oracle.quantize_tiles(q, seqs, 32, "q")
        kc = rng.integers(-127, 128, size=(32, 1, d), dtype=np.int8)
        ksc = (10.0 ** rng.uniform(-3, 0.5, size=(32, 1))).astype(np.float16)
        khat = oracle.dequant_cache(kc, ksc)[:, 0].astype(np.float64)
        sk = ksc[:, 0].astype(np.float64)
        s8 = float(qsc[0, 0]) * (qc[:, 0].astype(np.float64) @ kc[:, 0].astype(np.float64).T) * sk[None, :]
        s16 = q[:, 0].astype(np.float64) @ khat.T
        bound = d * float(qsc[0, 0]) * sk[None, :] * (127 / 2 + 127 ** 2 / 2 ** 11) * (1 + 2 ** -10)
        assert (np.abs(s8 - s16) <= bound).all()


def test_token_policy_threshold_is_inclusive_and_exact():
    # tau equal to fl32(s_q * mk) of the outlier's group routes it INT8; the
    # next fp32 value below routes it FP16 (the product is one fp32 rounding)
    tile, g = 32, 1
    seqs = oracle.seq_table(32, 128)
    qs = np.full((1, 2), np.float32(0.0123), dtype=np.float32)
    ktok = np.full((128, 1), 1e-3, dtype=np.float16)
    ktok[70, 0] = np.float16(0.7)
    t_eq = np.float32(np.float32(0.0123) * np.float32(np.float16(0.7)))
    m = oracle.build_mask_scale_policy(2, 1, seqs, tile, tile, g, False, qs, None, t_eq, k_token_scales=ktok)
    assert all(oracle.mask_bit(m, h, 0, G) == 1 for h in range(2) for G in range(4))
    t_lo = np.nextafter(t_eq, np.float32(0))
    m = oracle.build_mask_scale_policy(2, 1, seqs, tile, tile, g, False, qs, None, t_lo, k_token_scales=ktok)
    assert [oracle.mask_bit(m, 0, 0, G) for G in range(4)] == [1, 1, 0, 1]
