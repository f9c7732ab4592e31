"""GPU parity of the content-driven scale policy on the paths with their own
key offsets (prefix-cached prefill) and with an INT8 K/V cache, whose keys
carry one fp16 scale per token.

Bars: the key-tile statistic and the routing bits bit-exact against the
oracle for thresholds that split the groups, the extremes (tau = +inf and
tau < 0) and an outlier token placed by construction; the attention routed
by a policy mask within the attention tolerance of the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL, max_err
from mixed_precision_attention_tm_b200 import inputs, ops

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=[ops.ATTN_KERNEL_TWO_TILE, ops.ATTN_KERNEL_ONE_TILE],
                ids=["two_tile", "one_tile"])
def attn_kernel(request):
    ops.set_attn_kernel(request.param)
    yield request.param
    ops.set_attn_kernel(ops.ATTN_KERNEL_AUTO)


def _offsets(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def _taus(q_scales, k_stat):
    prods = np.outer(np.asarray(q_scales).ravel(), np.asarray(k_stat, dtype=np.float32).ravel()).ravel()
    return [float(np.quantile(prods, 0.9)), float(np.quantile(prods, 0.99)), float("inf"), -1.0]


def _tile_max(ks16, seqs, tile_n):
    """Largest token scale per (key tile, kv head), fp32: the reduction the
    device statistic must equal bit for bit."""
    kt = oracle.tile_table(seqs, tile_n, "k")
    out = np.zeros((len(kt), ks16.shape[1]), dtype=np.float32)
    for (_b, _i, r0, rows, ig) in kt:
        out[ig] = ks16[r0:r0 + rows].astype(np.float32).max(axis=0)
    return out


# (name, lq per sequence, lk per sequence or None for shared offsets, hq, hkv, causal, g, offsets)
CACHE_POLICY_CASES = [
    ("single_prefix", [300], [1000], 4, 2, True, 2, False),
    ("shared_varlen", [257, 640, 1], None, 4, 1, True, 1, True),
    ("key_offsets", [100, 256, 17], [900, 256, 400], 4, 2, True, 3, True),
    ("key_offsets_noncausal", [130, 60], [700, 129], 2, 1, False, 1, True),
]


@pytest.mark.parametrize("name,lq,lk,hq,hkv,causal,g,varlen", CACHE_POLICY_CASES,
                         ids=[c[0] for c in CACHE_POLICY_CASES])
def test_cache_scale_policy_bit_exact_and_attention(name, lq, lk, hq, hkv, causal, g, varlen):
    d, tm, tn = 128, 128, 128
    shared = lk is None
    lk = lq if shared else lk
    cu_q, cu_k = _offsets(lq), _offsets(lk)
    Tq, Tk = int(cu_q[-1]), int(cu_k[-1])
    q = inputs.randn_f16((Tq, hq, d), 60)
    k = inputs.randn_f16((Tk, hkv, d), 61)
    v = inputs.randn_f16((Tk, hkv, d), 62)
    # an outlier key token: 40x the values of one token of the middle key tile
    k[min(Tk - 1, Tk // 2 + 5)] *= 40
    kc, ks16 = inputs.int8_kv_cache(k)
    vc, vs16 = inputs.int8_kv_cache(v)
    if varlen:
        seqs = oracle.seq_table(Tq, Tk, cu_q, None if shared else cu_k)
        cq = torch.tensor(cu_q).cuda()
        ck = None if shared else torch.tensor(cu_k).cuda()
    else:
        seqs = oracle.seq_table(Tq, Tk)
        cq = ck = None
    qc, qs, _, _ = ops.quantize_qk(q.cuda(), None, tile_m=tm, tile_n=tn, cu_seqlens=cq)
    kstat = ops.key_tile_scales(ks16.cuda(), tile_n=tn, cu_seqlens_k=ck if ck is not None else cq)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    assert np.array_equal(kstat.cpu().numpy(), _tile_max(ks16.numpy(), seqs, tn))
    rq = oracle.quantize_tiles(q.numpy(), seqs, tm, "q")
    assert np.array_equal(qs.cpu().numpy(), rq[1])
    words = oracle.mask_words(max(lk), tn, g)
    kw = dict(tile_m=tm, tile_n=tn, g=g, causal=causal, force_diag=True, force_sink=False,
              Lq=Tq, Lk=Tk, cu_seqlens=cq, cu_seqlens_k=ck)
    split = 0
    for tau in _taus(rq[1], ks16.numpy()):
        m = ops.build_mask_scale_policy(qs, kstat, hq, hkv, tau=tau, **kw)
        torch.cuda.synchronize()
        assert ops.get_device_error() == ops.TM_OK
        ref = oracle.build_mask_scale_policy(hq, hkv, seqs, tm, tn, g, causal, rq[1], None, np.float32(tau),
                                             force_diag=True, words=words, k_token_scales=ks16.numpy())
        got = m.cpu().numpy().view(np.uint32)
        assert np.array_equal(got, ref), f"tau={tau}"
        full = oracle.build_mask(hq, seqs, tm, tn, g, causal, 1.0, 0, force_diag=True, words=words)
        split += int(ref.any() and not np.array_equal(ref, full))
    assert split >= 1
    # attention routed by the policy at the 0.99 quantile threshold
    tau = _taus(rq[1], ks16.numpy())[1]
    m = ops.build_mask_scale_policy(qs, kstat, hq, hkv, tau=tau, **kw)
    kv = tuple(t.cuda() for t in (kc, ks16, vc, vs16))
    out = ops.attn_fwd(q.cuda(), None, None, tile_m=tm, tile_n=tn, g=g, causal=causal, bitmask=m,
                       q_quant=(qc, qs), kv_cache=kv, cu_seqlens=cq, cu_seqlens_k=ck)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    mask_u32 = m.cpu().numpy().view(np.uint32)
    okw = dict(causal=causal, tile_m=tm, tile_n=tn, g=g, mask=mask_u32, q_quant=rq)
    if varlen:
        okw.update(cu_seqlens=cu_q, cu_seqlens_k=None if shared else cu_k)
    ref = oracle.attention(q.numpy(), kv_cache=(kc.numpy(), ks16.numpy(), vc.numpy(), vs16.numpy()), **okw)
    assert torch.isfinite(out).all()
    assert max_err(out.cpu(), ref) <= TOL


def test_key_offset_scale_policy_bit_exact_and_attention():
    # fp16 K with its own key offsets: tile scales from quantize_qk
    lq, lk = [77, 129, 0, 300], [300, 129, 520, 300]
    hq, hkv, d, tm, tn, g = 4, 2, 128, 128, 128, 2
    cu_q, cu_k = _offsets(lq), _offsets(lk)
    q, k, _ = inputs.qk_with_outliers(int(cu_q[-1]), int(cu_k[-1]), hq, hkv, d, 70)
    v = inputs.randn_f16((int(cu_k[-1]), hkv, d), 71)
    seqs = oracle.seq_table(len(q), len(k), cu_q, cu_k)
    cq, ck = torch.tensor(cu_q).cuda(), torch.tensor(cu_k).cuda()
    qc, qs, kc, ks = ops.quantize_qk(q.cuda(), k.cuda(), tile_m=tm, tile_n=tn, cu_seqlens=cq, cu_seqlens_k=ck)
    rq = oracle.quantize_tiles(q.numpy(), seqs, tm, "q")
    rk = oracle.quantize_tiles(k.numpy(), seqs, tn, "k")
    words = oracle.mask_words(max(lk), tn, g)
    kw = dict(tile_m=tm, tile_n=tn, g=g, causal=True, cu_seqlens=cq, cu_seqlens_k=ck, force_sink=True)
    for tau in _taus(rq[1], rk[1]):
        m = ops.build_mask_scale_policy(qs, ks, hq, hkv, tau=tau, **kw)
        torch.cuda.synchronize()
        ref = oracle.build_mask_scale_policy(hq, hkv, seqs, tm, tn, g, True, rq[1], rk[1], np.float32(tau),
                                             force_sink=True, words=words)
        assert np.array_equal(m.cpu().numpy().view(np.uint32), ref), f"tau={tau}"
    tau = float(np.quantile(np.outer(rq[1].ravel(), rk[1].ravel()), 0.5))
    m = ops.build_mask_scale_policy(qs, ks, hq, hkv, tau=tau, **kw)
    out = ops.attn_fwd(q.cuda(), k.cuda(), v.cuda(), tile_m=tm, tile_n=tn, g=g, causal=True, bitmask=m,
                       q_quant=(qc, qs), k_quant=(kc, ks), cu_seqlens=cq, cu_seqlens_k=ck)
    torch.cuda.synchronize()
    mask_u32 = m.cpu().numpy().view(np.uint32)
    ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), cu_seqlens=cu_q, cu_seqlens_k=cu_k, causal=True,
                           tile_m=tm, tile_n=tn, g=g, mask=mask_u32, q_quant=rq, k_quant=rk)
    assert max_err(out.cpu(), ref) <= TOL


def test_key_tile_scales_reports_a_key_sequence_beyond_its_bound():
    ks16 = torch.rand((512, 2), dtype=torch.float32).to(torch.float16).cuda()
    ck = torch.tensor([0, 100, 512], dtype=torch.int32).cuda()
    ops.key_tile_scales(ks16, tile_n=128, cu_seqlens_k=ck, max_seqlen_k=256)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_ERR_INVALID_ARG
    assert ops.get_device_error() == ops.TM_OK


def test_cache_policy_plan_matches_direct_calls():
    from mixed_precision_attention_tm_b200.api import TileMixPrefill
    lq, lk = [100, 256, 17], [900, 256, 400]
    hq, hkv, d = 4, 2, 128
    cu_q, cu_k = _offsets(lq), _offsets(lk)
    q = inputs.randn_f16((int(cu_q[-1]), hq, d), 80)
    k = inputs.randn_f16((int(cu_k[-1]), hkv, d), 81)
    v = inputs.randn_f16((int(cu_k[-1]), hkv, d), 82)
    kc, ks16 = inputs.int8_kv_cache(k)
    vc, vs16 = inputs.int8_kv_cache(v)
    tau = 2e-4
    pl = TileMixPrefill(int(cu_q[-1]), int(cu_k[-1]), hq, hkv, d, causal=True, g=2, tau=tau, int8_cache=True,
                        cu_seqlens=torch.tensor(cu_q), cu_seqlens_k=torch.tensor(cu_k))
    pl.load(q, kv_cache=(kc, ks16, vc, vs16))
    out = pl.run().clone()
    torch.cuda.synchronize()
    assert pl.launches_per_step == 5   # quantise Q, key statistic, mask, cache expansion, attention
    cq, ck = torch.tensor(cu_q).cuda(), torch.tensor(cu_k).cuda()
    qc, qs, _, _ = ops.quantize_qk(q.cuda(), None, cu_seqlens=cq)
    kstat = ops.key_tile_scales(ks16.cuda(), tile_n=128, cu_seqlens_k=ck)
    m = ops.build_mask_scale_policy(qs, kstat, hq, hkv, tile_m=128, tile_n=128, g=2, causal=True, tau=tau,
                                    cu_seqlens=cq, cu_seqlens_k=ck)
    assert torch.equal(pl.bitmask, m)
    kv = tuple(t.cuda() for t in (kc, ks16, vc, vs16))
    ws = torch.empty_like(pl.cache_ws)
    direct = ops.attn_fwd(q.cuda(), None, None, g=2, causal=True, bitmask=m, q_quant=(qc, qs), kv_cache=kv,
                          cu_seqlens=cq, cu_seqlens_k=ck, cache_workspace=ws)
    assert torch.equal(out, direct)
