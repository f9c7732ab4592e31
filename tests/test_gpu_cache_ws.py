"""GPU parity of the INT8-cache path with a caller workspace
(tm_attn_fwd_cache_ws): the cache's fp16 view and per-token K scales are
written once into the workspace, then the attention reads them.

Bars: the expanded fp16 K / V equal the oracle's fp16 view bit for bit and
the staged key-scale rows equal the cache's scales (zero past each
sequence's end); the attention output is within the attention tolerance of
the fp64 oracle, and equal bit for bit to the in-kernel conversion path
where both run on the two-query-tile kernel (routed launches).
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


# name, query lengths, key lengths (None: shared offsets; "single": one
# sequence without offsets), hq, hkv, causal, g, p (None: all FP16)
CASES = [
    ("varlen_routed", [300, 0, 800, 300], None, 4, 2, True, 2, 0.5),
    ("varlen_fp16", [257, 643], None, 4, 1, True, 1, None),
    ("single_all_int8", [700], "single", 2, 1, False, 1, 1.0),
    ("single_q_shorter", [300], [1000], 2, 2, True, 3, 0.5),
    ("prefix_routed", [100, 256, 17], [900, 256, 400], 8, 1, True, 2, 0.7),
    ("prefix_fp16", [200, 33], [1000, 700], 4, 2, False, 1, None),
    ("two_issuer_rows", [300, 8400], None, 2, 1, True, 4, 0.75),
]


def _run(case, seed=50):
    name, lq, lk, hq, hkv, causal, g, p = case
    d, tm, tn = 128, 128, 128
    single = lk == "single" or (lk is not None and len(lq) == 1 and name.startswith("single"))
    shared = lk is None or lk == "single"
    lk = lq if shared else lk
    cu_q, cu_k = _offsets(lq), _offsets(lk)
    Tq, Tk = int(cu_q[-1]), int(cu_k[-1])
    q = inputs.randn_f16((Tq, hq, d), seed)
    kc, ks16 = inputs.int8_kv_cache(inputs.randn_f16((Tk, hkv, d), seed + 1))
    vc, vs16 = inputs.int8_kv_cache(inputs.randn_f16((Tk, hkv, d), seed + 2))
    if single:
        seqs = oracle.seq_table(Tq, Tk)
        cq = ck = None
    else:
        seqs = oracle.seq_table(Tq, Tk, cu_q, None if shared else cu_k)
        cq = torch.tensor(cu_q).cuda()
        ck = None if shared else torch.tensor(cu_k).cuda()
    kv = tuple(t.cuda() for t in (kc, ks16, vc, vs16))
    qd = q.cuda()
    m = qq = None
    mask_u32 = None
    if p is not None:
        qc, qs, _, _ = ops.quantize_qk(qd, None, tile_m=tm, tile_n=tn, cu_seqlens=cq)
        qq = (qc, qs)
        if cq is None:
            m = ops.build_mask(hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed + 4, force_diag=True,
                               Lq=Tq, Lk=Tk)
        else:
            m = ops.build_mask(hq, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed + 4, force_diag=True,
                               cu_seqlens=cq, cu_seqlens_k=ck)
        torch.cuda.synchronize()
        mask_u32 = m.cpu().numpy().view(np.uint32)
    nb = 0 if cq is None else len(lq)
    ws = torch.empty(ops.cache_workspace_bytes(Tk, hkv, nb), dtype=torch.uint8, device="cuda")
    kw = dict(tile_m=tm, tile_n=tn, g=g, causal=causal, bitmask=m, q_quant=qq, kv_cache=kv, cu_seqlens=cq,
              cu_seqlens_k=ck)
    out_ws = ops.attn_fwd(qd, None, None, cache_workspace=ws, **kw)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    out_fused = ops.attn_fwd(qd, None, None, **kw)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    return dict(q=q, kc=kc, ks16=ks16, vc=vc, vs16=vs16, seqs=seqs, cu_q=None if cq is None else cu_q,
                cu_k=None if (cq is None or shared) else cu_k, mask=mask_u32, out_ws=out_ws.cpu(),
                out_fused=out_fused.cpu(), ws=ws, Tk=Tk, hkv=hkv, nb=nb, causal=causal, g=g, lq=lq)


def _rows(seqs, n_random=24, seed=5):
    rng = np.random.default_rng(seed)
    rows = set()
    for (qs, lq, _ks, _lk) in seqs:
        for r0 in range(0, lq, 128):
            rows.update([qs + r0, qs + min(lq, r0 + 128) - 1])
        if lq:
            rows.update(int(x) for x in rng.integers(qs, qs + lq, 4))
    return sorted(rows)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_cache_workspace_path_matches_oracle(case, attn_kernel):
    r = _run(case)
    big = sum(r["lq"]) > 4000
    rows = _rows(r["seqs"]) if big else None
    okw = dict(causal=r["causal"], tile_m=128, tile_n=128, g=r["g"], cu_seqlens=r["cu_q"], cu_seqlens_k=r["cu_k"])
    if r["mask"] is not None:
        okw.update(mask=r["mask"], q_quant=oracle.quantize_tiles(r["q"].numpy(), r["seqs"], 128, "q"))
    cache = tuple(t.numpy() for t in (r["kc"], r["ks16"], r["vc"], r["vs16"]))
    ref = oracle.attention(r["q"].numpy(), kv_cache=cache, rows=rows, **okw)
    assert torch.isfinite(r["out_ws"]).all()
    err = max_err(r["out_ws"], ref, rows=rows) if rows is not None else max_err(r["out_ws"], ref)
    assert err <= TOL, f"{case[0]}: max abs err {err}"
    # routed launches run the same scores and softmax on the two-query-tile
    # kernel either way: identical bits
    if r["mask"] is not None and attn_kernel == ops.ATTN_KERNEL_TWO_TILE:
        assert torch.equal(r["out_ws"], r["out_fused"])


def test_cache_workspace_holds_the_fp16_view_and_key_scale_rows(attn_kernel):
    r = _run(CASES[4])      # prefix_routed: separate key offsets, ragged key tiles
    ws = r["ws"].cpu().numpy()
    Tk, hkv, nb = r["Tk"], r["hkv"], r["nb"]
    kv_bytes = (Tk * hkv * 128 * 2 + 255) // 256 * 256
    k16 = ws[:Tk * hkv * 128 * 2].view(np.float16).reshape(Tk, hkv, 128)
    v16 = ws[kv_bytes:kv_bytes + Tk * hkv * 128 * 2].view(np.float16).reshape(Tk, hkv, 128)
    assert np.array_equal(k16.view(np.uint16), oracle.dequant_cache(r["kc"].numpy(), r["ks16"].numpy()).view(np.uint16))
    assert np.array_equal(v16.view(np.uint16), oracle.dequant_cache(r["vc"].numpy(), r["vs16"].numpy()).view(np.uint16))
    kst_tiles = (Tk + 127) // 128 + nb
    kst = ws[2 * kv_bytes:2 * kv_bytes + hkv * kst_tiles * 512].view(np.float32).reshape(hkv, kst_tiles, 128)
    ks = r["ks16"].numpy()
    for (b, _i, r0, rows, ig) in oracle.tile_table(r["seqs"], 128, "k"):
        want = np.zeros((hkv, 128), dtype=np.float32)
        want[:, :rows] = ks[r0:r0 + rows].T.astype(np.float32)
        assert np.array_equal(kst[:, ig].view(np.uint32), want.view(np.uint32)), (b, ig)


def test_cache_workspace_rejects_a_short_buffer():
    q = inputs.randn_f16((256, 2, 128), 1).cuda()
    kc, ks = inputs.int8_kv_cache(inputs.randn_f16((256, 1, 128), 2))
    kv = (kc.cuda(), ks.cuda(), kc.cuda(), ks.cuda())
    need = ops.cache_workspace_bytes(256, 1, 0)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        ops.attn_fwd(q, None, None, kv_cache=kv, causal=True, cache_workspace=ws)


def test_cache_workspace_reports_a_key_sequence_beyond_its_bound():
    cu_q = torch.tensor([0, 64], dtype=torch.int32).cuda()
    cu_k = torch.tensor([0, 512], dtype=torch.int32).cuda()
    q = inputs.randn_f16((64, 2, 128), 1).cuda()
    kc, ks = inputs.int8_kv_cache(inputs.randn_f16((512, 2, 128), 2))
    kv = (kc.cuda(), ks.cuda(), kc.cuda(), ks.cuda())
    ws = torch.empty(ops.cache_workspace_bytes(512, 2, 1), dtype=torch.uint8, device="cuda")
    ops.attn_fwd(q, None, None, kv_cache=kv, causal=True, cu_seqlens=cu_q, cu_seqlens_k=cu_k, max_seqlen=64,
                 max_seqlen_k=256, cache_workspace=ws)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_ERR_INVALID_ARG
    assert ops.get_device_error() == ops.TM_OK
