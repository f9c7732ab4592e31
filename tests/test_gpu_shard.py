"""Head-sharded prefill on one GPU: the interleaving copy against a plain
torch reference, and the sharded plan against the unsharded one.

Only one GPU is available to a test, so the ranks of a head-sharded problem
are emulated one after another: rank r's plan computes its query heads into
its slice, the slices are stacked as the all-gather would leave them, and
rank 0's plan interleaves them.  Every head is computed by the same kernels
on the same data whether or not the problem is sharded, so the result must
equal the unsharded plan's output bit for bit; one case is also held against
the fp64 oracle.  The collective itself is covered by the gloo test on CPU.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL
from mixed_precision_attention_tm_b200 import dist, inputs, ops
from mixed_precision_attention_tm_b200.api import HeadShardedPrefill, TileMixPrefill

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- the copy
@pytest.mark.parametrize("T,hq,world,d,pad", [(1, 1, 1, 64, 0), (257, 28, 8, 128, 0), (130, 6, 4, 64, 2),
                                              (64, 3, 8, 128, 0), (1000, 32, 3, 64, 1), (5, 65, 64, 8, 0)])
def test_merge_matches_reference(T, hq, world, d, pad):
    shards = dist.head_shards(hq, world)
    hs = [a for a, _ in shards] + [hq]
    h_cap = max(b - a for a, b in shards)
    gathered = inputs.randn_f16((world, T, h_cap, d), 5).cuda()
    buf = torch.full((T, hq + pad, d), -7.0, dtype=torch.float16, device="cuda")
    out = buf[:, :hq]                                   # strided rows when pad > 0
    ops.merge_head_shards(out, gathered, hs)
    torch.cuda.synchronize()
    ref = torch.empty((T, hq, d), dtype=torch.float16)
    g = gathered.cpu()
    for r, (a, b) in enumerate(shards):
        ref[:, a:b] = g[r, :, :b - a]
    assert torch.equal(out.cpu(), ref)
    if pad:
        assert bool((buf[:, hq:] == -7.0).all())        # nothing written past the heads


def test_merge_zero_rows():
    gathered = torch.empty((2, 0, 3, 64), dtype=torch.float16, device="cuda")
    out = torch.empty((0, 6, 64), dtype=torch.float16, device="cuda")
    ops.merge_head_shards(out, gathered, [0, 3, 6])
    torch.cuda.synchronize()


# ---------------------------------------------------------------- the plan
def _emulate(world, build, load_args):
    """Rank plans one after another on this GPU; returns rank 0's merged output."""
    plans = [build(rank=r, world=world) for r in range(world)]
    for pl in plans:
        pl.load(*load_args)
        pl.run_local()
    if world == 1:
        out = plans[0].run()
        torch.cuda.synchronize()
        return out.clone()
    for r, pl in enumerate(plans):
        plans[0].gathered[r].copy_(pl.out_local)
    plans[0].merge()
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    return plans[0].out.clone()


SHARD_CASES = [
    # name, Lq/Lk or cu, hq, hkv, d, g, mode, worlds
    ("gqa7_bernoulli", 1000, 28, 4, 128, 2, "p", (1, 3, 8)),
    ("gqa4_fp16", 700, 8, 2, 64, 1, "fp16", (2, 5)),
    ("gqa2_policy", 640, 6, 3, 128, 2, "tau", (4,)),
    ("varlen_cache", [0, 300, 1100, 1400], 8, 2, 128, 1, "cache", (3,)),
]


@pytest.mark.parametrize("case", SHARD_CASES, ids=[c[0] for c in SHARD_CASES])
def test_head_sharded_equals_unsharded(case):
    name, L, hq, hkv, d, g, mode, worlds = case
    cu = None
    if isinstance(L, list):
        cu = torch.tensor(L, dtype=torch.int32)
        L = L[-1]
    q = inputs.randn_f16((L, hq, d), 1).cuda()
    k16 = inputs.randn_f16((L, hkv, d), 2)
    v16 = inputs.randn_f16((L, hkv, d), 3)
    kw = dict(causal=True, tile_m=128, tile_n=128, g=g, force_diag=True, force_sink=True, cu_seqlens=cu)
    k = v = kv = None
    if mode == "cache":
        kc, ks = inputs.int8_kv_cache(k16)
        vc, vs = inputs.int8_kv_cache(v16)
        kv = tuple(t.cuda() for t in (kc, ks, vc, vs))
        kw.update(int8_cache=True, p=0.6, seed=9)
    else:
        k, v = k16.cuda(), v16.cuda()
        if mode == "p":
            kw.update(p=0.5, seed=9)
        elif mode == "tau":
            kw.update(tau=2e-4)
    base = TileMixPrefill(L, L, hq, hkv, d, **kw)
    base.load(q, k, v, kv)
    ref = base.run().clone()
    torch.cuda.synchronize()
    if mode in ("p", "cache"):
        bits = base.bitmask.cpu().numpy().view(np.uint32)
        assert bits.any() and not bits.all()              # both routes are taken
    for world in worlds:
        got = _emulate(world, lambda rank, world: HeadShardedPrefill(L, L, hq, hkv, d, rank=rank, world=world, **kw),
                       (q, k, v, kv))
        assert torch.equal(got, ref), f"world={world}"


def test_head_sharded_against_oracle():
    L, hq, hkv, d, g = 520, 6, 3, 64, 2
    q, k, v = (inputs.randn_f16((L, h, d), s) for h, s in ((hq, 21), (hkv, 22), (hkv, 23)))
    kw = dict(causal=True, tile_m=128, tile_n=128, g=g, p=0.5, seed=3, force_diag=True, force_sink=True)
    got = _emulate(4, lambda rank, world: HeadShardedPrefill(L, L, hq, hkv, d, rank=rank, world=world, **kw),
                   (q.cuda(), k.cuda(), v.cuda(), None))
    seqs = oracle.seq_table(L, L)
    mask = oracle.build_mask(hq, seqs, 128, 128, g, True, 0.5, 3, True, True)
    ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal=True, tile_m=128, tile_n=128, g=g, mask=mask,
                           q_quant=oracle.quantize_tiles(q.numpy(), seqs, 128, "q"),
                           k_quant=oracle.quantize_tiles(k.numpy(), seqs, 128, "k"))
    err = float(np.abs(got.cpu().double().numpy() - ref).max())
    assert err <= TOL, err


def test_plan_launch_count():
    pl = HeadShardedPrefill(256, 256, 28, 4, 128, rank=1, world=8, causal=True, g=2, p=0.5)
    # rank 1 holds heads 4..7: two segments (4..6 over KV head 0, 7 over KV head 1),
    # each quantising Q and K (one launch) and attending; one whole-problem
    # mask; one merge
    assert pl.segments == [(4, 7, 0, 1), (7, 8, 1, 2)]
    assert pl.launches_per_step == 2 * 2 + 1 + 1
