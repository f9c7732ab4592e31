"""The attention bindings refuse codes, scales and masks smaller than the
launch reads, and accept exactly what the library's producers allocate.

Runs on CPU: the binding code runs in full with CPU tensors, while the
library's device entry points are replaced by stubs that return TM_OK (the
host-side tile and word counts are the real library's).  Each case builds
its buffers through quantize_qk / quantize_qk_fp8 / build_mask, which
allocate them by their own sizing code, and hands them to attn_fwd /
attn_fwd_fp8."""

import pytest
import torch

from mixed_precision_attention_tm_b200 import inputs, ops

DEVICE_CALLS = ("tm_quantize_qk", "tm_quantize_qk_varlen", "tm_quantize_qk_fp8", "tm_build_mask",
                "tm_build_mask_varlen", "tm_build_mask_scale_policy", "tm_build_mask_scale_policy_varlen",
                "tm_key_tile_scales", "tm_attn_fwd", "tm_attn_fwd_varlen", "tm_attn_fwd_cache_ws",
                "tm_attn_fwd_fp8", "tm_merge_head_shards")


class _HostOnlyLib:
    def __init__(self, lib):
        self._lib = lib
        self.calls = []

    def __getattr__(self, name):
        if name in DEVICE_CALLS:
            def stub(*args):
                self.calls.append(name)
                return ops.TM_OK
            return stub
        return getattr(self._lib, name)


@pytest.fixture
def host_lib(monkeypatch):
    fake = _HostOnlyLib(ops._lib())
    monkeypatch.setattr(ops, "_lib", lambda: fake)
    monkeypatch.setattr(ops, "_cuda", lambda t, name: None)
    monkeypatch.setattr(ops, "_stream", lambda: None)
    return fake


def _qkv(Tq, Tk, hq, hkv, d):
    return (inputs.randn_f16((Tq, hq, d), 1), inputs.randn_f16((Tk, hkv, d), 2), inputs.randn_f16((Tk, hkv, d), 3))


CASES = [
    # Lq, Lk, hq, hkv, d, tile_m, tile_n, g, causal
    (1000, 1000, 4, 2, 128, 128, 128, 2, True),
    (300, 1000, 2, 2, 128, 128, 128, 1, True),
    (1000, 300, 2, 1, 128, 128, 128, 1, True),
    (600, 600, 2, 1, 128, 64, 128, 1, True),
    (600, 600, 2, 1, 128, 128, 64, 1, True),
    (256, 256, 2, 1, 64, 64, 64, 1, False),
    (50, 50, 1, 1, 128, 128, 128, 1, True),
    (256, 2051 * 128, 2, 1, 128, 128, 128, 1, True),
]


@pytest.mark.parametrize("case", CASES)
def test_producer_buffers_are_accepted_and_short_ones_refused(host_lib, case):
    Lq, Lk, hq, hkv, d, tm, tn, g, causal = case
    q, k, v = _qkv(Lq, Lk, hq, hkv, d)
    qc, qs, kc, ks = ops.quantize_qk(q, k, tile_m=tm, tile_n=tn)
    m = ops.build_mask(hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=0.5, seed=1, Lq=Lq, Lk=Lk, device="cpu")
    kw = dict(tile_m=tm, tile_n=tn, g=g, causal=causal)
    ops.attn_fwd(q, k, v, bitmask=m, q_quant=(qc, qs), k_quant=(kc, ks), **kw)
    ops.attn_fwd(q, k, v, bitmask=m[:1], q_quant=(qc, qs), k_quant=(kc, ks), **kw)   # one shared plane
    ops.attn_fwd(q, k, v, **kw)                                                    # all FP16
    assert host_lib.calls.count("tm_attn_fwd") == 3
    short = [
        dict(bitmask=m.flatten()[:-1].view(1, 1, -1)[..., :], q_quant=(qc, qs), k_quant=(kc, ks)),
        dict(bitmask=m, q_quant=(qc, qs.flatten()[:-1]), k_quant=(kc, ks)),
        dict(bitmask=m, q_quant=(qc, qs), k_quant=(kc, ks.flatten()[:-1])),
        dict(bitmask=m, q_quant=(qc.flatten()[:-1], qs), k_quant=(kc, ks)),
        dict(bitmask=m, q_quant=(qc.to(torch.uint8), qs), k_quant=(kc, ks)),
        dict(bitmask=m, q_quant=(qc, qs.double()), k_quant=(kc, ks)),
    ]
    for i, bad in enumerate(short):
        with pytest.raises(ValueError):
            ops.attn_fwd(q, k, v, mask_head_stride=m.shape[1] * m.shape[2] if i == 0 else None, **bad, **kw)
    assert host_lib.calls.count("tm_attn_fwd") == 3       # nothing short reached the library


def test_varlen_prefix_shards_cache_and_fp8(host_lib):
    # shared offsets
    cu = torch.tensor([0, 300, 300, 1100, 1400], dtype=torch.int32)
    q, k, v = _qkv(1400, 1400, 4, 2, 128)
    qc, qs, kc, ks = ops.quantize_qk(q, k, cu_seqlens=cu)
    m = ops.build_mask(4, tile_m=128, tile_n=128, g=2, causal=True, p=0.5, seed=1, cu_seqlens=cu, device="cpu")
    ops.attn_fwd(q, k, v, g=2, causal=True, bitmask=m, q_quant=(qc, qs), k_quant=(kc, ks), cu_seqlens=cu)
    with pytest.raises(ValueError):
        ops.attn_fwd(q, k, v, g=2, causal=True, bitmask=m, q_quant=(qc, qs[:-1]), k_quant=(kc, ks), cu_seqlens=cu)
    # separate key offsets (prefix-cached prefill), key maximum computed or declared
    cq = torch.tensor([0, 64, 300], dtype=torch.int32)
    ckk = torch.tensor([0, 512, 1400], dtype=torch.int32)
    q2, k2, v2 = _qkv(300, 1400, 2, 2, 128)
    qc2, qs2, kc2, ks2 = ops.quantize_qk(q2, k2, cu_seqlens=cq, cu_seqlens_k=ckk)
    m2 = ops.build_mask(2, tile_m=128, tile_n=128, g=1, causal=True, p=0.5, seed=2, cu_seqlens=cq,
                        cu_seqlens_k=ckk, device="cpu")
    kw2 = dict(g=1, causal=True, bitmask=m2, q_quant=(qc2, qs2), k_quant=(kc2, ks2), cu_seqlens=cq,
               cu_seqlens_k=ckk)
    ops.attn_fwd(q2, k2, v2, **kw2)
    ops.attn_fwd(q2, k2, v2, max_seqlen=236, max_seqlen_k=888, **kw2)
    assert host_lib.calls.count("tm_attn_fwd_varlen") == 2
    # head-sharded segments read slices of the whole problem's mask
    mfull = ops.build_mask(8, tile_m=128, tile_n=128, g=1, causal=True, p=0.5, seed=3, Lq=700, Lk=700, device="cpu")
    q3, k3, v3 = _qkv(700, 700, 3, 1, 128)
    qc3, qs3, kc3, ks3 = ops.quantize_qk(q3, k3)
    ops.attn_fwd(q3, k3, v3, causal=True, bitmask=mfull[4:7], q_quant=(qc3, qs3), k_quant=(kc3, ks3))
    # INT8 K/V cache: no K tile scales
    kcache, kscale = inputs.int8_kv_cache(k3)
    vcache, vscale = inputs.int8_kv_cache(v3)
    ops.attn_fwd(q3, None, None, causal=True, bitmask=mfull[4:7], q_quant=(qc3, qs3),
                 kv_cache=(kcache, kscale, vcache, vscale))
    # FP8 route: both planes and both code sets
    qf = ops.quantize_qk_fp8(q3, k3)
    mf = ops.build_mask(3, tile_m=128, tile_n=128, g=1, causal=True, p=0.5, seed=4, Lq=700, Lk=700, device="cpu")
    m8 = ops.build_mask(3, tile_m=128, tile_n=128, g=1, causal=True, p=0.5, seed=5, Lq=700, Lk=700, device="cpu")
    ops.attn_fwd_fp8(q3, k3, v3, causal=True, bitmask_fp8=mf, qf8_quant=qf[:2], kf8_quant=qf[2:])
    ops.attn_fwd_fp8(q3, k3, v3, causal=True, bitmask_fp8=mf, qf8_quant=qf[:2], kf8_quant=qf[2:], bitmask=m8,
                     q_quant=(qc3, qs3), k_quant=(kc3, ks3))
    with pytest.raises(ValueError):
        ops.attn_fwd_fp8(q3, k3, v3, causal=True, bitmask_fp8=mf, qf8_quant=(qf[0], qf[1][:-1]), kf8_quant=qf[2:])
    with pytest.raises(ValueError):
        ops.attn_fwd_fp8(q3, k3, v3, causal=True, bitmask_fp8=mf, qf8_quant=(qc3, qs3), kf8_quant=qf[2:])
    assert host_lib.calls.count("tm_attn_fwd_fp8") == 2


PLANS = [
    # name, Lq/Lk or (cu, cu_k), hq, hkv, plan keywords
    ("routed", 1000, 4, 2, dict(g=2, p=0.5, force_diag=True, force_sink=True)),
    ("policy", 1000, 4, 2, dict(g=2, tau=1e-3)),
    ("fp16", 700, 8, 2, dict()),
    ("varlen_cache", ([0, 300, 1100, 1400], None), 8, 2, dict(p=0.6, int8_cache=True)),
    ("prefix_cache", ([0, 64, 300], [0, 512, 1400]), 2, 2, dict(p=0.75, int8_cache=True)),
    ("prefix_fp16_keys", ([0, 64, 300], [0, 512, 1400]), 2, 2, dict(p=0.75)),
]


def _plan_inputs(L, hq, hkv, kw):
    cu = ck = None
    if isinstance(L, tuple):
        cu, ck = (None if x is None else torch.tensor(x, dtype=torch.int32) for x in L)
        Lq, Lk = int(cu[-1]), int((ck if ck is not None else cu)[-1])
    else:
        Lq = Lk = L
    q, k, v = _qkv(Lq, Lk, hq, hkv, 128)
    kv = None
    if kw.get("int8_cache"):
        kv = (*inputs.int8_kv_cache(k), *inputs.int8_kv_cache(v))
        k = v = None
    return Lq, Lk, cu, ck, q, k, v, kv


@pytest.mark.parametrize("plan", PLANS, ids=[p[0] for p in PLANS])
def test_plans_pass_the_checks(host_lib, plan):
    from mixed_precision_attention_tm_b200.api import HeadShardedPrefill, TileMixPrefill
    name, L, hq, hkv, kw = plan
    Lq, Lk, cu, ck, q, k, v, kv = _plan_inputs(L, hq, hkv, kw)
    common = dict(causal=True, cu_seqlens=cu, cu_seqlens_k=ck, device="cpu", **kw)
    pl = TileMixPrefill(Lq, Lk, hq, hkv, 128, **common)
    pl.load(q, k, v, kv)
    pl.run()
    if ck is None:                 # head sharding takes shared offsets
        for world in (1, 3):
            for rank in range(world):
                sp = HeadShardedPrefill(Lq, Lk, hq, hkv, 128, rank=rank, world=world,
                                        **{x: y for x, y in common.items() if x != "cu_seqlens_k"})
                sp.load(q, k, v, kv)
                sp.run_local()
    assert any(c in host_lib.calls for c in ("tm_attn_fwd", "tm_attn_fwd_varlen", "tm_attn_fwd_cache_ws"))
