"""GPU parity: the CUDA path (through the C-ABI) against the fp64 oracle on
identical seeded inputs.

Bars: INT8 codes, tile scales and routing bits bit-exact; attention output
max-abs error <= 3e-3 (fp16 output, unit-variance inputs).  Sizes span
several tiles and a ragged tail while the oracle still finishes in seconds.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL, max_err, oracle_mask, run_gpu, run_oracle, seqs_of
from mixed_precision_attention_tm_b200 import inputs, ops

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=[ops.ATTN_KERNEL_TWO_TILE, ops.ATTN_KERNEL_ONE_TILE],
                ids=["two_tile", "one_tile"])
def attn_kernel(request):
    """Every case runs through both d = 128 attention kernels (the two-tile
    and the one-tile kernel); other launches are unaffected by the choice."""
    ops.set_attn_kernel(request.param)
    yield request.param
    ops.set_attn_kernel(ops.ATTN_KERNEL_AUTO)


def W(Lq, Lk, hq, hkv, d, causal, tm=128, tn=128, g=1, p=None, seed=0, fd=False, fs=False,
      outliers=False, cu=None):
    if cu is not None:
        cu_t = torch.tensor(cu, dtype=torch.int32)
        lens = cu_t[1:] - cu_t[:-1]
        Lq = Lk = int(cu[-1])
    else:
        cu_t = lens = None
    if outliers:
        q, k, _ = inputs.qk_with_outliers(Lq, Lk, hq, hkv, d, seed)
    else:
        q, k = inputs.randn_f16((Lq, hq, d), seed), inputs.randn_f16((Lk, hkv, d), seed + 1)
    v = inputs.randn_f16((Lk, hkv, d), seed + 2)
    return inputs.Workload(f"w{Lq}x{Lk}", q, k, v, hq, hkv, d, causal, tm, tn, g, p, mask_seed=seed + 4,
                           force_diag=fd, force_sink=fs, cu_seqlens=cu_t, lens=lens)


# ------------------------------------------------------------------ quantiser
QUANT_CASES = [
    # (T, H, d, tile, cu, scale)
    (256, 2, 64, 64, None, 1.0),
    (1000, 4, 128, 128, None, 1.0),
    (777, 3, 64, 128, None, 20.0),
    (1400, 2, 128, 64, [0, 300, 300, 1100, 1400], 1.0),
    (50, 1, 128, 128, None, 1e-3),
]


@pytest.mark.parametrize("case", QUANT_CASES)
def test_quantizer_bit_exact(case):
    T, H, d, tile, cu, scale = case
    x = inputs.randn_f16((T, H, d), 7, scale)
    x[3:5] = 0                                    # zeros inside a tile
    if T >= 256:
        x[tile:2 * tile, 0] = 0                   # an all-zero (tile, head) block
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    maxlen = None if cu is None else max(b - a for a, b in zip(cu[:-1], cu[1:]))
    qc, qs, _, _ = ops.quantize_qk(x.cuda(), None, tile_m=tile, tile_n=tile, cu_seqlens=cu_t, max_seqlen=maxlen)
    torch.cuda.synchronize()
    seqs = oracle.seq_table(T, T, cu)
    rc, rs = oracle.quantize_tiles(x.numpy(), seqs, tile, "q")
    assert np.array_equal(qs.cpu().numpy(), rs)
    assert np.array_equal(qc.cpu().numpy(), rc)


def test_quantizer_q_and_k_tiles_differ():
    q = inputs.randn_f16((500, 4, 128), 1)
    k = inputs.randn_f16((500, 2, 128), 2)
    qc, qs, kc, ks = ops.quantize_qk(q.cuda(), k.cuda(), tile_m=64, tile_n=128)
    torch.cuda.synchronize()
    seqs = oracle.seq_table(500, 500)
    rqc, rqs = oracle.quantize_tiles(q.numpy(), seqs, 64, "q")
    rkc, rks = oracle.quantize_tiles(k.numpy(), seqs, 128, "k")
    assert np.array_equal(qs.cpu().numpy(), rqs) and np.array_equal(qc.cpu().numpy(), rqc)
    assert np.array_equal(ks.cpu().numpy(), rks) and np.array_equal(kc.cpu().numpy(), rkc)


def test_quantizer_ties_and_near_ties_bit_exact():
    """Tiles whose values sit exactly on, or within 2^-13 of, the half-integer
    boundaries of rne(fl32(x / s)) (power-of-two and other scales, Q and K in
    one launch, d = 64 and 128): codes and scales equal the oracle's."""
    from quant_cases import AMAXES, tie_tile
    for d in (64, 128):
        tiles = [tie_tile(128, d, np.float16(a), i) for i, a in enumerate(AMAXES)]
        x = np.stack(tiles, axis=1).reshape(128, len(AMAXES), d)            # heads = amax cases
        q = torch.from_numpy(np.concatenate([x, x[::-1]], axis=0).copy())   # two tiles per head
        k = torch.from_numpy(x[:, ::-1].copy())
        qc, qs, kc, ks = ops.quantize_qk(q.cuda(), k.cuda(), tile_m=128, tile_n=128)
        torch.cuda.synchronize()
        rqc, rqs = oracle.quantize_tiles(q.numpy(), oracle.seq_table(256, 256), 128, "q")
        rkc, rks = oracle.quantize_tiles(k.numpy(), oracle.seq_table(128, 128), 128, "k")
        assert np.array_equal(qs.cpu().numpy(), rqs) and np.array_equal(ks.cpu().numpy(), rks)
        assert np.array_equal(qc.cpu().numpy(), rqc) and np.array_equal(kc.cpu().numpy(), rkc)


# ------------------------------------------------------------------ mask
MASK_CASES = [
    # (Hq, Lq, Lk, cu, tm, tn, g, causal, p, fd, fs)
    (2, 256, 256, None, 64, 64, 1, False, 0.5, False, False),
    (32, 16384, 16384, None, 128, 128, 4, True, 0.75, True, True),
    (3, 700, 2100, None, 128, 64, 3, True, 0.4, True, False),
    (4, 1500, 300, None, 64, 128, 1, True, 0.9, False, True),
    (5, 0, 0, [0, 1000, 1000, 5000, 5001], 128, 128, 4, True, 0.75, True, True),
    (28, 65536, 65536, None, 128, 128, 8, True, 0.5, True, True),
]


@pytest.mark.parametrize("case", MASK_CASES)
def test_device_mask_bit_exact(case):
    Hq, Lq, Lk, cu, tm, tn, g, causal, p, fd, fs = case
    seed = 1234 + Hq
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")
    m = ops.build_mask(Hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed, force_diag=fd,
                       force_sink=fs, Lq=Lq, Lk=Lk, cu_seqlens=cu_t)
    torch.cuda.synchronize()
    got = m.cpu().numpy().view(np.uint32)
    if cu is not None:
        Lq = Lk = cu[-1]
    ref = oracle.build_mask(Hq, oracle.seq_table(Lq, Lk, cu), tm, tn, g, causal, p, seed, fd, fs)
    assert np.array_equal(got, ref)
    host = ops.build_mask_host(Hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed,
                               force_diag=fd, force_sink=fs, Lq=Lq, Lk=Lk, cu_seqlens_host=cu)
    assert np.array_equal(got, host)


# ------------------------------------------------------------------ attention vs oracle
ATTN_CASES = [
    # id, workload kwargs
    ("tiny_fp16", dict(Lq=256, Lk=256, hq=2, hkv=1, d=64, causal=False, tm=64, tn=64)),
    ("tiny_int8_half", dict(Lq=256, Lk=256, hq=2, hkv=1, d=64, causal=False, tm=64, tn=64, p=0.5)),
    ("d128_causal_ragged", dict(Lq=1000, Lk=1000, hq=4, hkv=2, d=128, causal=True)),
    ("d128_noncausal_ragged", dict(Lq=1000, Lk=1000, hq=4, hkv=2, d=128, causal=False)),
    ("d64_causal_ragged", dict(Lq=1000, Lk=1000, hq=4, hkv=1, d=64, causal=True)),
    ("d128_routed_g2", dict(Lq=1000, Lk=1000, hq=4, hkv=2, d=128, causal=True, g=2, p=0.5, fd=True, fs=True)),
    ("d128_all_int8", dict(Lq=700, Lk=700, hq=2, hkv=1, d=128, causal=False, p=1.0)),
    ("d64_routed", dict(Lq=900, Lk=900, hq=4, hkv=2, d=64, causal=True, p=0.6)),
    ("q_shorter", dict(Lq=300, Lk=1000, hq=2, hkv=2, d=128, causal=True, p=0.5)),
    ("q_longer_empty_rows", dict(Lq=1000, Lk=300, hq=2, hkv=1, d=128, causal=True, p=0.5)),
    ("tm64_tn128", dict(Lq=600, Lk=600, hq=2, hkv=1, d=128, causal=True, tm=64, tn=128, p=0.5)),
    ("tm128_tn64", dict(Lq=600, Lk=600, hq=2, hkv=1, d=128, causal=True, tm=128, tn=64, p=0.5)),
    ("d64_tn128_tm64", dict(Lq=600, Lk=600, hq=2, hkv=1, d=64, causal=False, tm=64, tn=128, p=0.5)),
    ("outliers_routed", dict(Lq=1024, Lk=1024, hq=4, hkv=1, d=128, causal=True, g=4, p=0.75, fd=True, fs=True,
                              outliers=True)),
    ("varlen_routed", dict(Lq=0, Lk=0, hq=4, hkv=2, d=128, causal=True, g=2, p=0.5, fd=True, fs=True,
                           cu=[0, 300, 300, 1100, 1400])),
    ("varlen_fp16_noncausal", dict(Lq=0, Lk=0, hq=2, hkv=1, d=64, causal=False, cu=[0, 129, 200, 457])),
    ("short_T", dict(Lq=50, Lk=50, hq=1, hkv=1, d=128, causal=True, p=0.5)),
    ("single_token", dict(Lq=1, Lk=1, hq=2, hkv=1, d=64, causal=True)),
]


@pytest.mark.parametrize("name,kw", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attention_matches_oracle(name, kw):
    w = W(**kw)
    out, m, quant = run_gpu(w)
    mask_u32 = None if m is None else m.numpy().view(np.uint32)
    if mask_u32 is not None:
        assert np.array_equal(mask_u32, oracle_mask(w))        # device bits == oracle bits
        seqs, _ = seqs_of(w)
        rqc, rqs = oracle.quantize_tiles(w.q.numpy(), seqs, w.tile_m, "q")
        assert np.array_equal(quant[1].numpy(), rqs) and np.array_equal(quant[0].numpy(), rqc)
    ref = run_oracle(w, mask_u32)
    assert torch.isfinite(out).all()
    err = max_err(out, ref)
    assert err <= TOL, f"{name}: max abs err {err}"


def test_long_key_rows_read_routing_words_and_scales_from_global_memory():
    """Key rows of 2051 tiles at g = 1 need 65 routing words: both kernels keep
    64 words and the first 256 (two-tile) or 512 (one-tile) key-tile scales in
    shared memory, and read the rest from global memory."""
    Lk = 2051 * 128
    assert ops.mask_words(Lk, 128, 1) > 64
    w = W(Lq=256, Lk=Lk, hq=2, hkv=1, d=128, causal=True, g=1, p=0.5, fd=True, fs=True)
    out, m, _ = run_gpu(w)
    mask_u32 = m.numpy().view(np.uint32)
    assert np.array_equal(mask_u32, oracle_mask(w))
    rows = [0, 1, 63, 127, 128, 129, 200, 255]
    ref = run_oracle(w, mask_u32, rows=rows)
    err = max_err(out, ref, rows=rows)
    assert err <= TOL, f"max abs err {err}"


# ------------------------------------------------------------------ GPU invariants
def test_lossless_inputs_route_invisible_on_gpu():
    L, hq, hkv, d = 640, 2, 1, 128
    q, k = inputs.lossless_qk([(0, L)], [(0, L)], L, L, hq, hkv, d, 128, 128, seed=3)
    v = inputs.randn_f16((L, hkv, d), 5)
    base = inputs.Workload("ll", q, k, v, hq, hkv, d, True, 128, 128, 1, None)
    routed = inputs.Workload("ll", q, k, v, hq, hkv, d, True, 128, 128, 1, 0.6, mask_seed=9)
    o0, _, _ = run_gpu(base)
    o1, m, _ = run_gpu(routed)
    assert m.numpy().any()
    # INT8 and FP16 scores are the same numbers here, so the outputs agree bit for bit
    assert torch.equal(o0, o1)


def test_constant_values_give_ones():
    w = W(Lq=800, Lk=800, hq=2, hkv=1, d=128, causal=True, p=0.5)
    w.v = torch.ones_like(w.v)
    out, _, _ = run_gpu(w)
    assert (out.float() - 1).abs().max().item() <= 2e-3


def test_gqa_equals_repeated_heads_on_gpu():
    w = W(Lq=640, Lk=640, hq=8, hkv=2, d=128, causal=True, p=0.5)
    o1, m, _ = run_gpu(w)
    w2 = W(Lq=640, Lk=640, hq=8, hkv=2, d=128, causal=True, p=0.5)
    w2.k = w.k.repeat_interleave(4, dim=1)
    w2.v = w.v.repeat_interleave(4, dim=1)
    w2.hkv = 8
    o2, _, _ = run_gpu(w2, mask=m.numpy().view(np.uint32))
    assert torch.equal(o1, o2)


def test_varlen_equals_separate_calls_on_gpu():
    cu = [0, 300, 300, 1100, 1400]
    w = W(Lq=0, Lk=0, hq=4, hkv=2, d=128, causal=True, g=2, p=0.5, cu=cu)
    whole, m, _ = run_gpu(w)
    mask = m.numpy().view(np.uint32)
    qt0 = 0
    for b in range(len(cu) - 1):
        a, e = cu[b], cu[b + 1]
        n = oracle.n_tiles(e - a, 128)
        sub = mask[:, qt0:qt0 + n, :]
        qt0 += n
        if e == a:
            continue
        wb = inputs.Workload("part", w.q[a:e].clone(), w.k[a:e].clone(), w.v[a:e].clone(), 4, 2, 128, True,
                             128, 128, 2, 0.5)
        part, _, _ = run_gpu(wb, mask=np.ascontiguousarray(sub[:, :, :oracle.mask_words(e - a, 128, 2)]))
        assert torch.equal(whole[a:e], part), b


def test_grouping_equals_replicated_bits_on_gpu():
    w = W(Lq=1024, Lk=1024, hq=2, hkv=1, d=128, causal=True, g=3, p=0.5)
    o3, m, _ = run_gpu(w)
    mg = m.numpy().view(np.uint32)
    nkt = 1024 // 128
    m1 = np.zeros((2, mg.shape[1], 1), dtype=np.uint32)
    for h in range(2):
        for I in range(mg.shape[1]):
            for J in range(nkt):
                if oracle.mask_bit(mg, h, I, J // 3):
                    m1[h, I, 0] |= np.uint32(1 << J)
    w1 = W(Lq=1024, Lk=1024, hq=2, hkv=1, d=128, causal=True, g=1, p=0.5)
    o1, _, _ = run_gpu(w1, mask=m1)
    assert torch.equal(o3, o1)


def test_shared_mask_plane_on_gpu():
    w = W(Lq=512, Lk=512, hq=4, hkv=1, d=128, causal=False, p=0.5)
    seqs, _ = seqs_of(w)
    one = oracle.build_mask(1, seqs, 128, 128, 1, False, 0.5, 77)
    o_shared, _, _ = run_gpu(w, mask=one)
    o_full, _, _ = run_gpu(w, mask=np.repeat(one, 4, axis=0))
    assert torch.equal(o_shared, o_full)


def test_deterministic():
    w = W(Lq=1000, Lk=1000, hq=4, hkv=2, d=128, causal=True, p=0.5)
    a, _, _ = run_gpu(w)
    b, _, _ = run_gpu(w)
    assert torch.equal(a, b)


def test_noncontiguous_head_strides():
    # Q / K / V as slices of one packed [T, Hq + 2 Hkv, d] projection output
    L, hq, hkv, d = 700, 4, 2, 128
    packed = inputs.randn_f16((L, hq + 2 * hkv, d), 21)
    q, k, v = packed[:, :hq], packed[:, hq:hq + hkv], packed[:, hq + hkv:]
    pc = packed.cuda()
    out = ops.attn_fwd(pc[:, :hq], pc[:, hq:hq + hkv], pc[:, hq + hkv:], causal=True)
    torch.cuda.synchronize()
    ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal=True)
    assert max_err(out.cpu(), ref) <= TOL


# ------------------------------------------------------------------ INT8 K/V cache
def Wc(hq, hkv, causal, p=None, g=1, tm=128, cu=None, Lq=None, Lk=None, seed=0, fd=False, fs=False):
    if cu is not None:
        cu_t = torch.tensor(cu, dtype=torch.int32)
        lens = cu_t[1:] - cu_t[:-1]
        Lq = Lk = int(cu[-1])
    else:
        cu_t = lens = None
    d = 128
    q = inputs.randn_f16((Lq, hq, d), seed)
    k = inputs.randn_f16((Lk, hkv, d), seed + 1)
    v = inputs.randn_f16((Lk, hkv, d), seed + 2)
    kc, ks = inputs.int8_kv_cache(k)
    vc, vs = inputs.int8_kv_cache(v)
    return inputs.Workload("cache", q, None, None, hq, hkv, d, causal, tm, 128, g, p, mask_seed=seed + 4,
                           force_diag=fd, force_sink=fs, cu_seqlens=cu_t, lens=lens, kv_cache=(kc, ks, vc, vs))


CACHE_CASES = [
    ("varlen_cache_routed", dict(hq=4, hkv=2, causal=True, p=0.5, g=2, cu=[0, 300, 300, 1100, 1400], fd=True, fs=True)),
    ("varlen_cache_fp16", dict(hq=4, hkv=1, causal=True, p=None, cu=[0, 257, 900])),
    ("cache_all_int8", dict(hq=2, hkv=1, causal=False, p=1.0, Lq=700, Lk=700)),
    ("cache_q_shorter", dict(hq=2, hkv=2, causal=True, p=0.5, Lq=300, Lk=1000)),
    ("cache_tm64", dict(hq=2, hkv=1, causal=True, p=0.5, tm=64, Lq=600, Lk=600)),
]


@pytest.mark.parametrize("name,kw", CACHE_CASES, ids=[c[0] for c in CACHE_CASES])
def test_int8_cache_matches_oracle(name, kw):
    w = Wc(**kw)
    out, m, _ = run_gpu(w)
    mask_u32 = None if m is None else m.numpy().view(np.uint32)
    if mask_u32 is not None:
        assert np.array_equal(mask_u32, oracle_mask(w))
    ref = run_oracle(w, mask_u32)
    assert torch.isfinite(out).all()
    err = max_err(out, ref)
    assert err <= TOL, f"{name}: max abs err {err}"


def test_int8_cache_fp16_route_equals_dequantised_fp16_inputs():
    # With every group FP16, the cache path must equal the fp16 path fed with
    # the cache's fp16 view fp16(code * scale) (the same numbers reach the MMAs).
    w = Wc(hq=4, hkv=2, causal=True, p=None, Lq=640, Lk=640)
    out_c, _, _ = run_gpu(w)
    kc, ks, vc, vs = w.kv_cache
    k16 = torch.from_numpy(oracle.dequant_cache(kc.numpy(), ks.numpy()))
    v16 = torch.from_numpy(oracle.dequant_cache(vc.numpy(), vs.numpy()))
    wf = inputs.Workload("f", w.q, k16, v16, 4, 2, 128, True, 128, 128, 1, None)
    out_f, _, _ = run_gpu(wf)
    assert max_err(out_c, out_f.to(torch.float64).numpy()) <= 2e-3


# ------------------------------------------------------------------ two-issuer mode
# Rows of 64 or more key tiles run the 128x128 kernel with one tcgen05 issuer
# per query tile (shorter rows share one issuer); these cases reach that mode
# with an absent second query tile, ragged key tails, causal rows of different
# lengths, varlen batches mixing long and short sequences, and d = 64.
DUAL_CASES = [
    ("dual_noncausal_tileB_absent", dict(Lq=384, Lk=8269, hq=2, hkv=1, d=128, causal=False, g=2, p=0.5)),
    ("dual_causal_ragged_outliers", dict(Lq=8269, Lk=8269, hq=2, hkv=1, d=128, causal=True, g=1, p=0.5,
                                         fd=True, fs=True, outliers=True)),
    ("dual_causal_fp16", dict(Lq=8205, Lk=8205, hq=2, hkv=2, d=128, causal=True)),
    # all-FP16 launches with rows of 64 key tiles or more take the chunked
    # two-tile mode (64-key chunks in two score slots per query tile)
    ("dual_noncausal_fp16_gqa_ragged", dict(Lq=300, Lk=8269, hq=4, hkv=2, d=128, causal=False)),
    ("dual_varlen_fp16", dict(Lq=0, Lk=0, hq=2, hkv=1, d=128, causal=True, cu=[0, 8300, 8500])),
    ("dual_varlen_mixed", dict(Lq=0, Lk=0, hq=4, hkv=2, d=128, causal=True, g=4, p=0.75,
                               cu=[0, 300, 8500, 8629, 8800])),
    ("dual_d64", dict(Lq=320, Lk=8192, hq=2, hkv=1, d=64, causal=False, g=1, p=1.0)),
]


def _rows_for(w, seed=5, n_random=40):
    seqs, _ = seqs_of(w)
    rng = np.random.default_rng(seed)
    rows = set()
    for (qs, lq, _ks, _lk) in seqs:
        if lq == 0:
            continue
        for r0 in range(0, lq, 128):      # first and last row of every query tile
            rows.update([qs + r0, qs + min(lq, r0 + 128) - 1])
        rows.update(int(x) for x in rng.integers(qs, qs + lq, max(1, n_random // len(seqs))))
    return sorted(rows)


@pytest.mark.parametrize("name,kw", DUAL_CASES, ids=[c[0] for c in DUAL_CASES])
def test_two_issuer_mode_matches_oracle(name, kw):
    w = W(**kw)
    out, m, _ = run_gpu(w)
    assert torch.isfinite(out).all()
    mask_u32 = None if m is None else m.numpy().view(np.uint32)
    if mask_u32 is not None:
        assert np.array_equal(mask_u32, oracle_mask(w))
    rows = _rows_for(w)
    ref = run_oracle(w, mask_u32, rows=rows)
    err = max_err(out, ref, rows=rows)
    assert err <= TOL, f"{name}: max abs err {err} over {len(rows)} rows"


# ------------------------------------------------------------------ scale policy
POLICY_CASES = [
    dict(Lq=700, Lk=700, hq=4, hkv=2, d=128, causal=True, g=2, tm=128, tn=128, fd=True, fs=True, outliers=True),
    dict(Lq=300, Lk=900, hq=2, hkv=1, d=64, causal=False, g=1, tm=64, tn=64, outliers=True),
    dict(Lq=0, Lk=0, hq=4, hkv=1, d=128, causal=True, g=3, cu=[0, 130, 600, 1000], outliers=True),
]


@pytest.mark.parametrize("kw", POLICY_CASES, ids=["causal_gqa", "noncausal_64", "varlen"])
def test_scale_policy_mask_bit_exact_and_attention(kw):
    w = W(**kw)
    seqs, cu = seqs_of(w)
    q, k = w.q.cuda(), w.k.cuda()
    cu_d = None if w.cu_seqlens is None else w.cu_seqlens.cuda()
    ms = w.max_seqlen if cu is not None else None
    qc, qs, kc, ks = ops.quantize_qk(q, k, tile_m=w.tile_m, tile_n=w.tile_n, cu_seqlens=cu_d, max_seqlen=ms)
    rq = oracle.quantize_tiles(w.q.numpy(), seqs, w.tile_m, "q")[1]
    rk = oracle.quantize_tiles(w.k.numpy(), seqs, w.tile_n, "k")[1]
    prods = np.sort(np.outer(rq.ravel(), rk.ravel()).ravel())
    for tau in (float(np.quantile(prods, 0.3)), float(np.quantile(prods, 0.8)), float("inf"), -1.0):
        m = ops.build_mask_scale_policy(qs, ks, w.hq, w.hkv, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g,
                                        causal=w.causal, tau=tau, force_diag=w.force_diag, force_sink=w.force_sink,
                                        Lq=w.Lq, Lk=w.Lk, cu_seqlens=cu_d, max_seqlen=ms)
        torch.cuda.synchronize()
        ref = oracle.build_mask_scale_policy(w.hq, w.hkv, seqs, w.tile_m, w.tile_n, w.g, w.causal, rq, rk,
                                             np.float32(tau), force_diag=w.force_diag, force_sink=w.force_sink)
        got = m.cpu().numpy().view(np.uint32)
        assert np.array_equal(got, ref), f"tau={tau}"
    # the attention with the last non-trivial policy mask matches the oracle
    tau = float(np.quantile(prods, 0.5))
    m = ops.build_mask_scale_policy(qs, ks, w.hq, w.hkv, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g,
                                    causal=w.causal, tau=tau, force_diag=w.force_diag, force_sink=w.force_sink,
                                    Lq=w.Lq, Lk=w.Lk, cu_seqlens=cu_d, max_seqlen=ms)
    out, _, _ = run_gpu(w, mask=m.cpu().numpy().view(np.uint32))
    ref = run_oracle(w, m.cpu().numpy().view(np.uint32))
    assert max_err(out, ref) <= TOL


def test_scale_policy_plan_matches_direct_calls():
    from mixed_precision_attention_tm_b200.api import TileMixPrefill
    w = W(Lq=1000, Lk=1000, hq=4, hkv=2, d=128, causal=True, g=2, outliers=True)
    pl = TileMixPrefill(w.Lq, w.Lk, w.hq, w.hkv, w.d, causal=True, g=2, tau=1e-3)
    pl.load(w.q, w.k, w.v)
    out = pl.run().clone()
    torch.cuda.synchronize()
    qc, qs, kc, ks = ops.quantize_qk(w.q.cuda(), w.k.cuda())
    m = ops.build_mask_scale_policy(qs, ks, 4, 2, tile_m=128, tile_n=128, g=2, causal=True, tau=1e-3,
                                    Lq=w.Lq, Lk=w.Lk)
    direct = ops.attn_fwd(w.q.cuda(), w.k.cuda(), w.v.cuda(), g=2, causal=True, bitmask=m,
                          q_quant=(qc, qs), k_quant=(kc, ks))
    assert torch.equal(out, direct)


# ------------------------------------------------------------------ separate key offsets
# Prefix-cached prefill: sequence b has lq new queries and lk >= lq keys
# (cu_seqlens_k), bottom-right causal per sequence; fp16 K/V through the
# 128x128 pair kernel and the 64-row single-tile kernel, and an INT8 cache.
PREFIX_CASES = [
    ("pair_causal", dict(lq=[77, 129, 0, 300], lk=[300, 129, 520, 300], hq=4, hkv=2, d=128, causal=True,
                         tm=128, tn=128, g=2, p=0.6)),
    ("pair_noncausal_fp16", dict(lq=[200, 33], lk=[1000, 700], hq=2, hkv=1, d=64, causal=False,
                                 tm=128, tn=128, g=1, p=None)),
    ("single_tile_64", dict(lq=[90, 64], lk=[250, 64], hq=2, hkv=2, d=128, causal=True, tm=64, tn=64, g=1, p=0.5)),
    ("int8_cache", dict(lq=[100, 256, 17], lk=[900, 256, 400], hq=4, hkv=1, d=128, causal=True, tm=128, tn=128,
                        g=2, p=0.7, cache=True)),
]


@pytest.mark.parametrize("name,kw", PREFIX_CASES, ids=[c[0] for c in PREFIX_CASES])
def test_prefix_prefill_matches_oracle(name, kw):
    lq, lk = kw["lq"], kw["lk"]
    hq, hkv, d, causal, tm, tn, g, p = kw["hq"], kw["hkv"], kw["d"], kw["causal"], kw["tm"], kw["tn"], kw["g"], kw["p"]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    q = inputs.randn_f16((int(cu_q[-1]), hq, d), 40)
    k = inputs.randn_f16((int(cu_k[-1]), hkv, d), 41)
    v = inputs.randn_f16((int(cu_k[-1]), hkv, d), 42)
    seqs = oracle.seq_table(len(q), len(k), cu_q, cu_k)
    cq, ck = torch.tensor(cu_q).cuda(), torch.tensor(cu_k).cuda()
    kv = None
    if kw.get("cache"):
        kc, ks16 = inputs.int8_kv_cache(k)
        vc, vs16 = inputs.int8_kv_cache(v)
        kv = (kc, ks16, vc, vs16)
    qd = q.cuda()
    kd = None if kv is not None else k.cuda()
    qc, qs, kcd, ksd = ops.quantize_qk(qd, kd, tile_m=tm, tile_n=tn, cu_seqlens=cq, cu_seqlens_k=ck)
    m = mask_u32 = None
    if p is not None:
        m = ops.build_mask(hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=9, force_diag=True,
                           cu_seqlens=cq, cu_seqlens_k=ck)
        torch.cuda.synchronize()
        mask_u32 = m.cpu().numpy().view(np.uint32)
        assert np.array_equal(mask_u32, oracle.build_mask(hq, seqs, tm, tn, g, causal, p, 9, force_diag=True))
        rq = oracle.quantize_tiles(q.numpy(), seqs, tm, "q")
        assert np.array_equal(qs.cpu().numpy(), rq[1]) and np.array_equal(qc.cpu().numpy(), rq[0])
        if kv is None:
            rk = oracle.quantize_tiles(k.numpy(), seqs, tn, "k")
            assert np.array_equal(ksd.cpu().numpy(), rk[1]) and np.array_equal(kcd.cpu().numpy(), rk[0])
    out = ops.attn_fwd(qd, kd, None if kv is not None else v.cuda(), tile_m=tm, tile_n=tn, g=g, causal=causal,
                       bitmask=m, q_quant=(qc, qs) if m is not None else None,
                       k_quant=(kcd, ksd) if (m is not None and kv is None) else None,
                       kv_cache=None if kv is None else tuple(t.cuda() for t in kv),
                       cu_seqlens=cq, cu_seqlens_k=ck)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    okw = dict(cu_seqlens=cu_q, cu_seqlens_k=cu_k, causal=causal, tile_m=tm, tile_n=tn, g=g)
    if mask_u32 is not None:
        okw.update(mask=mask_u32, q_quant=oracle.quantize_tiles(q.numpy(), seqs, tm, "q"))
        if kv is None:
            okw["k_quant"] = oracle.quantize_tiles(k.numpy(), seqs, tn, "k")
    if kv is not None:
        ref = oracle.attention(q.numpy(), kv_cache=tuple(t.numpy() for t in kv), **okw)
    else:
        ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), **okw)
    assert max_err(out.cpu(), ref) <= TOL


def test_prefix_prefill_longer_keys_than_declared_is_reported():
    cu_q = torch.tensor([0, 64], dtype=torch.int32).cuda()
    cu_k = torch.tensor([0, 512], dtype=torch.int32).cuda()
    q = inputs.randn_f16((64, 2, 128), 1).cuda()
    k = inputs.randn_f16((512, 2, 128), 2).cuda()
    v = inputs.randn_f16((512, 2, 128), 3).cuda()
    ops.attn_fwd(q, k, v, causal=True, cu_seqlens=cu_q, cu_seqlens_k=cu_k, max_seqlen=64, max_seqlen_k=256)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_ERR_INVALID_ARG
    assert ops.get_device_error() == ops.TM_OK          # reading clears the word
