"""Pins of the oracle's tile-routed attention.

Sources: TileMix (Lattice paper page), abstract (routing per score-tile
group, FP16 or INT8 scores, shared softmax, dense connectivity, GQA, varlen,
INT8 K/V cache); MLX PR "Nax Refactor" attention tables (fp16 fused SDPA,
GQA, causal).  Each test pins the oracle to something other than itself: a
scalar brute force, a library routine (fp64 torch SDPA), a closed form or an
invariant of the mathematics.
"""


import numpy as np
import pytest
import torch

import oracle
from bruteforce import brute_attention
from mixed_precision_attention_tm_b200 import inputs


def _f16(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def _quant(q, k, seqs, tm, tn):
    return (oracle.quantize_tiles(q, seqs, tm, "q"), oracle.quantize_tiles(k, seqs, tn, "k"))


def _run(q, k, v, cu=None, causal=False, tm=2, tn=2, g=1, mask=None, cache=None):
    Tq = q.shape[0]
    Tk = (k if cache is None else cache[0]).shape[0]
    seqs = oracle.seq_table(Tq, Tk, cu)
    kw = dict(cu_seqlens=cu, causal=causal, tile_m=tm, tile_n=tn, g=g)
    if mask is not None:
        qq = oracle.quantize_tiles(q, seqs, tm, "q")
        kq = None if cache is not None else oracle.quantize_tiles(k, seqs, tn, "k")
        kw.update(mask=mask, q_quant=qq, k_quant=kq, kv_cache=cache)
    elif cache is not None:
        kw.update(kv_cache=cache)
    return oracle.attention(q, None if cache is not None else k, None if cache is not None else v, **kw)


BRUTE_CASES = [
    # (Lq, Lk, cu, Hq, Hkv, d, causal, tm, tn, g, p)
    (6, 6, None, 1, 1, 4, False, 2, 2, 1, None),
    (6, 6, None, 2, 1, 4, True, 2, 2, 1, 0.5),
    (5, 8, None, 2, 2, 3, True, 2, 3, 2, 0.6),
    (8, 5, None, 4, 2, 4, True, 3, 2, 1, 0.5),          # Lq > Lk: empty rows
    (7, 7, None, 2, 1, 4, False, 3, 2, 2, 1.0),
    (0, 0, [0, 3, 3, 8], 2, 1, 4, True, 2, 2, 1, 0.5),  # varlen with an empty sequence
    (0, 0, [0, 5, 9], 3, 1, 2, False, 2, 3, 1, 0.7),
]


@pytest.mark.parametrize("case", BRUTE_CASES)
@pytest.mark.parametrize("seed", [0, 1])
def test_matches_scalar_bruteforce(case, seed):
    Lq, Lk, cu, Hq, Hkv, d, causal, tm, tn, g, p = case
    if cu is not None:
        Lq = Lk = cu[-1]
    rng = np.random.default_rng(seed)
    q = _f16(rng, (Lq, Hq, d), 2.0)
    k = _f16(rng, (Lk, Hkv, d), 2.0)
    v = _f16(rng, (Lk, Hkv, d))
    seqs = oracle.seq_table(Lq, Lk, cu)
    mask = None
    if p is not None:
        mask = oracle.build_mask(Hq, seqs, tm, tn, g, causal, p, 1000 + seed)
    got = _run(q, k, v, cu, causal, tm, tn, g, mask)
    bits = None if mask is None else (lambda h, I, G: oracle.mask_bit(mask, h, I, G))
    ref = brute_attention(q.astype(float).tolist(), k.astype(float).tolist(), v.astype(float).tolist(),
                          Hq, Hkv, d, causal, tm, tn, g, bits, cu)
    np.testing.assert_allclose(got, np.array(ref), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_int8_cache_matches_scalar_bruteforce(seed):
    rng = np.random.default_rng(seed)
    cu = [0, 4, 9]
    T, Hq, Hkv, d, tm, tn, g = 9, 2, 1, 4, 2, 2, 1
    q = _f16(rng, (T, Hq, d), 2.0)
    kc = rng.integers(-127, 128, (T, Hkv, d)).astype(np.int8)
    vc = rng.integers(-127, 128, (T, Hkv, d)).astype(np.int8)
    ks = (rng.random((T, Hkv)) * 0.05).astype(np.float16)
    vs = (rng.random((T, Hkv)) * 0.05).astype(np.float16)
    cache = (kc, ks, vc, vs)
    seqs = oracle.seq_table(T, T, cu)
    mask = oracle.build_mask(Hq, seqs, tm, tn, g, True, 0.5, 7 + seed)
    got = _run(q, None, None, cu, True, tm, tn, g, mask, cache=cache)
    k16 = oracle.dequant_cache(kc, ks)
    v16 = oracle.dequant_cache(vc, vs)
    # the fp16 view is fp16(code * scale) with the product exact in fp32
    assert np.array_equal(k16, (kc.astype(np.float64) * ks.astype(np.float64)[..., None]).astype(np.float16))
    ref = brute_attention(q.astype(float).tolist(), k16.astype(float).tolist(), v16.astype(float).tolist(),
                          Hq, Hkv, d, True, tm, tn, g, lambda h, I, G: oracle.mask_bit(mask, h, I, G), cu,
                          cache=(kc.astype(int).tolist(), ks.astype(float).tolist()))
    np.testing.assert_allclose(got, np.array(ref), rtol=1e-12, atol=1e-12)


def _sdpa_fp64(q, k, v, causal):
    """Library reference: torch SDPA in fp64 on CPU, bottom-right causal mask,
    KV heads repeated for GQA."""
    Lq, Hq, d = q.shape
    Lk, Hkv, _ = k.shape
    Q = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)
    K = torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    V = torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    attn_mask = None
    if causal:
        i = torch.arange(Lq)[:, None]
        j = torch.arange(Lk)[None, :]
        attn_mask = j <= i + (Lk - Lq)
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=attn_mask)
    return O.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Lq,Lk,Hq,Hkv,d,causal", [
    (300, 300, 4, 2, 64, False), (300, 300, 4, 1, 64, True),
    (129, 517, 2, 2, 128, True), (200, 200, 8, 2, 128, True),
])
def test_all_fp16_equals_library_sdpa(Lq, Lk, Hq, Hkv, d, causal):
    rng = np.random.default_rng(Lq + Lk)
    q, k, v = _f16(rng, (Lq, Hq, d)), _f16(rng, (Lk, Hkv, d)), _f16(rng, (Lk, Hkv, d))
    got = _run(q, k, v, None, causal, 64, 64, 1, None)
    ref = _sdpa_fp64(q, k, v, causal)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
    # an all-zero mask is the same computation
    seqs = oracle.seq_table(Lq, Lk)
    zero = oracle.build_mask(Hq, seqs, 64, 64, 1, causal, 0.0, 0)
    got0 = _run(q, k, v, None, causal, 64, 64, 1, zero)
    np.testing.assert_array_equal(got0, got)


@pytest.mark.parametrize("causal", [False, True])
def test_lossless_inputs_make_routing_invisible(causal):
    L, Hq, Hkv, d, tm, tn = 256, 2, 1, 64, 64, 64
    qt, kt = inputs.lossless_qk([(0, L)], [(0, L)], L, L, Hq, Hkv, d, tm, tn, seed=11)
    q, k = qt.numpy(), kt.numpy()
    v = _f16(np.random.default_rng(0), (L, Hkv, d))
    seqs = oracle.seq_table(L, L)
    (qc, qs), (kc, ks) = _quant(q, k, seqs, tm, tn)
    assert np.all(qs == np.float32(2.0 ** -6)) and np.all(ks == np.float32(2.0 ** -6))
    assert np.array_equal(qc.astype(np.float64) * 2.0 ** -6, q.astype(np.float64))
    base = _run(q, k, v, None, causal, tm, tn, 1, None)
    for p in (0.5, 1.0):
        mask = oracle.build_mask(Hq, seqs, tm, tn, 1, causal, p, 3)
        got = _run(q, k, v, None, causal, tm, tn, 1, mask)
        np.testing.assert_allclose(got, base, rtol=1e-12, atol=1e-13)


def test_int8_route_differs_without_lossless_inputs():
    # guards against a mask that is silently ignored
    rng = np.random.default_rng(5)
    L, d = 128, 64
    q, k, v = _f16(rng, (L, 1, d), 3.0), _f16(rng, (L, 1, d), 3.0), _f16(rng, (L, 1, d))
    seqs = oracle.seq_table(L, L)
    mask = oracle.build_mask(1, seqs, 64, 64, 1, False, 1.0, 0)
    a = _run(q, k, v, None, False, 64, 64, 1, None)
    b = _run(q, k, v, None, False, 64, 64, 1, mask)
    assert np.abs(a - b).max() > 1e-4


@pytest.mark.parametrize("p", [0.0, 0.5, 1.0])
def test_constant_values_give_constant_output(p):
    rng = np.random.default_rng(9)
    Lq, Lk, Hq, Hkv, d = 150, 190, 4, 2, 32
    q, k = _f16(rng, (Lq, Hq, d), 4.0), _f16(rng, (Lk, Hkv, d), 4.0)
    v = np.ones((Lk, Hkv, d), dtype=np.float16)
    seqs = oracle.seq_table(Lq, Lk)
    mask = oracle.build_mask(Hq, seqs, 32, 32, 2, True, p, 1)
    got = _run(q, k, v, None, True, 32, 32, 2, mask)
    np.testing.assert_allclose(got, 1.0, rtol=0, atol=1e-12)


def test_probability_rows_sum_to_one():
    # V = identity (d == Lk) exposes P itself as the output
    rng = np.random.default_rng(2)
    L, d = 16, 16
    q, k = _f16(rng, (L, 1, d), 3.0), _f16(rng, (L, 1, d), 3.0)
    v = np.eye(L, dtype=np.float16).reshape(L, 1, d)
    seqs = oracle.seq_table(L, L)
    mask = oracle.build_mask(1, seqs, 4, 4, 1, True, 0.5, 4)
    P = _run(q, k, v, None, True, 4, 4, 1, mask)[:, 0, :]
    assert np.all(P >= 0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(np.triu(P, 1) == 0)                  # causal: no future key


def test_causal_rows_ignore_future_keys():
    rng = np.random.default_rng(4)
    Lq, Lk, Hq, d = 96, 160, 2, 32
    q, k, v = _f16(rng, (Lq, Hq, d)), _f16(rng, (Lk, 1, d)), _f16(rng, (Lk, 1, d))
    base = _run(q, k, v, None, True, 32, 32, 1, None)
    for i in (0, 17, 95):
        jcut = i + Lk - Lq                              # last visible key of row i
        k2, v2 = k.copy(), v.copy()
        k2[jcut + 1:] = _f16(rng, k2[jcut + 1:].shape, 5.0)
        v2[jcut + 1:] = _f16(rng, v2[jcut + 1:].shape, 5.0)
        got = _run(q, k2, v2, None, True, 32, 32, 1, None)
        np.testing.assert_array_equal(got[i], base[i])
    # square causal: row 0 sees only key 0
    sq = _run(q[:64], k[:64], v[:64], None, True, 32, 32, 1, None)
    np.testing.assert_allclose(sq[0, :, :], np.repeat(v[0:1, 0, :].astype(np.float64), Hq, 0), atol=0)


def test_empty_rows_are_zero():
    rng = np.random.default_rng(6)
    Lq, Lk = 40, 10
    q, k, v = _f16(rng, (Lq, 1, 8)), _f16(rng, (Lk, 1, 8)), _f16(rng, (Lk, 1, 8))
    got = _run(q, k, v, None, True, 8, 8, 1, None)
    assert np.all(got[:Lq - Lk] == 0)
    assert np.all(np.abs(got[Lq - Lk:]).sum(axis=-1) > 0)


@pytest.mark.parametrize("p", [None, 0.6])
def test_gqa_equals_repeated_kv_heads(p):
    rng = np.random.default_rng(8)
    L, Hq, Hkv, d, t = 200, 6, 2, 32, 32
    q, k, v = _f16(rng, (L, Hq, d), 3.0), _f16(rng, (L, Hkv, d), 3.0), _f16(rng, (L, Hkv, d))
    seqs = oracle.seq_table(L, L)
    mask = None if p is None else oracle.build_mask(Hq, seqs, t, t, 1, True, p, 2)
    a = _run(q, k, v, None, True, t, t, 1, mask)
    kr, vr = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    b = _run(q, kr, vr, None, True, t, t, 1, mask)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("p", [None, 0.5])
def test_varlen_equals_separate_calls(p):
    rng = np.random.default_rng(10)
    cu = [0, 70, 70, 231, 300]
    T, Hq, Hkv, d, t, g = cu[-1], 4, 2, 32, 32, 2
    q, k, v = _f16(rng, (T, Hq, d), 3.0), _f16(rng, (T, Hkv, d), 3.0), _f16(rng, (T, Hkv, d))
    seqs = oracle.seq_table(T, T, cu)
    mask = None if p is None else oracle.build_mask(Hq, seqs, t, t, g, True, p, 5)
    whole = _run(q, k, v, cu, True, t, t, g, mask)
    qt0 = 0
    for b in range(len(cu) - 1):
        a, e = cu[b], cu[b + 1]
        nqt = oracle.n_tiles(e - a, t)
        sub = None if mask is None else mask[:, qt0:qt0 + nqt, :]
        qt0 += nqt
        if e == a:
            continue
        part = _run(q[a:e], k[a:e], v[a:e], None, True, t, t, g, sub)
        np.testing.assert_array_equal(whole[a:e], part)


def test_grouping_equals_replicated_bits():
    rng = np.random.default_rng(12)
    L, Hq, d, t, g = 256, 2, 32, 32, 3
    q, k, v = _f16(rng, (L, Hq, d), 3.0), _f16(rng, (L, 1, d), 3.0), _f16(rng, (L, 1, d))
    seqs = oracle.seq_table(L, L)
    mg = oracle.build_mask(Hq, seqs, t, t, g, True, 0.5, 8)
    nkt = oracle.n_tiles(L, t)
    m1 = np.zeros((Hq, mg.shape[1], oracle.mask_words(L, t, 1)), dtype=np.uint32)
    for h in range(Hq):
        for I in range(mg.shape[1]):
            for J in range(nkt):
                if oracle.mask_bit(mg, h, I, J // g):
                    m1[h, I, J // 32] |= np.uint32(1 << (J % 32))
    a = _run(q, k, v, None, True, t, t, g, mg)
    b = _run(q, k, v, None, True, t, t, 1, m1)
    np.testing.assert_array_equal(a, b)


def test_shared_mask_head_plane():
    rng = np.random.default_rng(13)
    L, Hq, d, t = 128, 3, 16, 32
    q, k, v = _f16(rng, (L, Hq, d), 3.0), _f16(rng, (L, 1, d), 3.0), _f16(rng, (L, 1, d))
    seqs = oracle.seq_table(L, L)
    m = oracle.build_mask(1, seqs, t, t, 1, False, 0.5, 1)
    a = _run(q, k, v, None, False, t, t, 1, m)
    b = _run(q, k, v, None, False, t, t, 1, np.repeat(m, Hq, axis=0))
    np.testing.assert_array_equal(a, b)


def test_sampled_rows_match_full():
    rng = np.random.default_rng(14)
    L, Hq, d = 300, 2, 32
    q, k, v = _f16(rng, (L, Hq, d)), _f16(rng, (L, 1, d)), _f16(rng, (L, 1, d))
    seqs = oracle.seq_table(L, L)
    mask = oracle.build_mask(Hq, seqs, 64, 64, 1, True, 0.5, 3)
    (qq, kq) = _quant(q, k, seqs, 64, 64)
    full = oracle.attention(q, k, v, causal=True, tile_m=64, tile_n=64, mask=mask, q_quant=qq, k_quant=kq)
    rows = [0, 63, 64, 200, 299]
    part = oracle.attention_rows(q, k, v, rows=rows, causal=True, tile_m=64, tile_n=64, mask=mask,
                                 q_quant=qq, k_quant=kq)
    np.testing.assert_allclose(part[rows], full[rows], rtol=1e-12, atol=1e-14)
    assert np.isnan(part[1]).all()


# ------------------------------------------------------------------ separate key offsets
# Prefix-cached prefill (cu_seqlens_k != cu_seqlens): sequence b's lq new query
# tokens attend to its lk >= lq keys, prefix first, bottom-right causal.

def test_prefix_prefill_equals_last_rows_of_full_self_attention():
    rng = np.random.default_rng(21)
    lk_list, lq_list = [300, 129, 520], [77, 129, 5]
    Hq, Hkv, d = 4, 2, 32
    # full sequences: K, V of lk tokens; the new queries are the last lq rows of Q_full
    qf = [rng.standard_normal((lk, Hq, d)).astype(np.float16) for lk in lk_list]
    kf = [rng.standard_normal((lk, Hkv, d)).astype(np.float16) for lk in lk_list]
    vf = [rng.standard_normal((lk, Hkv, d)).astype(np.float16) for lk in lk_list]
    q = np.concatenate([x[-lq:] for x, lq in zip(qf, lq_list)])
    k, v = np.concatenate(kf), np.concatenate(vf)
    cu_q = np.concatenate([[0], np.cumsum(lq_list)])
    cu_k = np.concatenate([[0], np.cumsum(lk_list)])
    for causal in (True, False):
        got = oracle.attention(q, k, v, cu_seqlens=cu_q, cu_seqlens_k=cu_k, causal=causal, tile_m=32, tile_n=32)
        for b, (lq, lk) in enumerate(zip(lq_list, lk_list)):
            full = oracle.attention(qf[b], kf[b], vf[b], causal=causal, tile_m=32, tile_n=32)
            np.testing.assert_allclose(got[cu_q[b]:cu_q[b + 1]], full[lk - lq:], rtol=0, atol=1e-12)


def test_prefix_prefill_routed_equals_per_sequence_calls():
    rng = np.random.default_rng(22)
    lq_list, lk_list = [40, 100], [200, 100]
    Hq, Hkv, d = 2, 1, 16
    q = rng.standard_normal((sum(lq_list), Hq, d)).astype(np.float16)
    k = rng.standard_normal((sum(lk_list), Hkv, d)).astype(np.float16)
    v = rng.standard_normal((sum(lk_list), Hkv, d)).astype(np.float16)
    cu_q = np.concatenate([[0], np.cumsum(lq_list)])
    cu_k = np.concatenate([[0], np.cumsum(lk_list)])
    seqs = oracle.seq_table(len(q), len(k), cu_q, cu_k)
    assert seqs == [(0, 40, 0, 200), (40, 100, 200, 100)]
    mask = oracle.build_mask(Hq, seqs, 32, 32, 2, True, 0.6, 5, force_diag=True)
    qq = oracle.quantize_tiles(q, seqs, 32, "q")
    kq = oracle.quantize_tiles(k, seqs, 32, "k")
    got = oracle.attention(q, k, v, cu_seqlens=cu_q, cu_seqlens_k=cu_k, causal=True, tile_m=32, tile_n=32, g=2,
                           mask=mask, q_quant=qq, k_quant=kq)
    qt0 = 0
    for b, (lq, lk) in enumerate(zip(lq_list, lk_list)):
        qb, kb, vb = q[cu_q[b]:cu_q[b + 1]], k[cu_k[b]:cu_k[b + 1]], v[cu_k[b]:cu_k[b + 1]]
        sb = oracle.seq_table(lq, lk)
        nqt = oracle.n_tiles(lq, 32)
        mb = oracle.build_mask(Hq, sb, 32, 32, 2, True, 0.6, 5, force_diag=True)
        # the batched mask rows of this sequence carry the batched hash keys (I_glob); reuse them
        mb[:, :, :] = mask[:, qt0:qt0 + nqt, :mb.shape[2]]
        ref = oracle.attention(qb, kb, vb, causal=True, tile_m=32, tile_n=32, g=2, mask=mb,
                               q_quant=oracle.quantize_tiles(qb, sb, 32, "q"),
                               k_quant=oracle.quantize_tiles(kb, sb, 32, "k"))
        np.testing.assert_allclose(got[cu_q[b]:cu_q[b + 1]], ref, rtol=0, atol=1e-12)
        qt0 += nqt
