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
