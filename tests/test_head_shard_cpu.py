"""Head-sharded prefill on CPU: the host logic of splitting one problem by
query heads over ranks, and its all-gather, over world-size-2 gloo ranks.

Each rank evaluates its heads with the oracle, segment by segment exactly as
the GPU plan calls the library (query heads [s0, s1) over KV heads [k0, k1),
the routing bits of the whole problem sliced by head), gathers the
equal-size slices with ``dist.all_gather_heads`` and interleaves them; the
result must equal the oracle's unsharded output bit for bit, since every
head is computed by the same operations either way.  The interleaving copy
of the product is a CUDA kernel (tm_merge_head_shards), checked on the GPU;
here only its argument validation runs (it fails before any CUDA call)."""

import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from mixed_precision_attention_tm_b200 import dist, inputs, ops


# ---------------------------------------------------------------- partition
@pytest.mark.parametrize("hq,world", [(32, 1), (32, 8), (28, 8), (28, 3), (6, 4), (3, 8), (1, 2)])
def test_head_shards_cover_and_balance(hq, world):
    sh = dist.head_shards(hq, world)
    assert len(sh) == world
    assert sh[0][0] == 0 and sh[-1][1] == hq
    assert all(a <= b for a, b in sh) and all(sh[i][1] == sh[i + 1][0] for i in range(world - 1))
    sizes = [b - a for a, b in sh]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == hq


@pytest.mark.parametrize("hq,hkv,world", [(32, 8, 8), (28, 4, 8), (28, 4, 3), (6, 3, 2), (6, 3, 4), (12, 1, 5),
                                          (8, 8, 3)])
def test_kv_segments_keep_the_gqa_map(hq, hkv, world):
    grp = hq // hkv
    for h0, h1 in dist.head_shards(hq, world):
        segs = dist.kv_segments(h0, h1, grp)
        covered = []
        for s0, s1, k0, k1 in segs:
            assert s1 > s0 and k1 > k0
            n_q, n_k = s1 - s0, k1 - k0
            assert n_q % n_k == 0
            g_loc = n_q // n_k
            # the library's map inside the segment equals the global one
            for hl in range(n_q):
                assert k0 + hl // g_loc == (s0 + hl) // grp
            # a segment with several KV heads holds whole groups only
            if n_k > 1:
                assert g_loc == grp and s0 % grp == 0
            covered.extend(range(s0, s1))
        assert covered == list(range(h0, h1))


def test_kv_segments_examples():
    # 28 query heads over 4 KV heads (7 per group), rank 1 of 8 holds heads 4..7
    assert dist.kv_segments(4, 8, 7) == [(4, 7, 0, 1), (7, 8, 1, 2)]
    assert dist.kv_segments(0, 32, 4) == [(0, 32, 0, 8)]
    assert dist.kv_segments(2, 10, 4) == [(2, 4, 0, 1), (4, 8, 1, 2), (8, 10, 2, 3)]
    assert dist.kv_segments(5, 5, 4) == []


# ---------------------------------------------------------------- gloo ranks
CASE = dict(L=200, hq=6, hkv=3, d=64, tile=64, g=2, p=0.5, causal=True, seed=11)


def _problem():
    c = CASE
    q, k = inputs.randn_f16((c["L"], c["hq"], c["d"]), c["seed"]), inputs.randn_f16((c["L"], c["hkv"], c["d"]),
                                                                                     c["seed"] + 1)
    v = inputs.randn_f16((c["L"], c["hkv"], c["d"]), c["seed"] + 2)
    seqs = oracle.seq_table(c["L"], c["L"])
    mask = oracle.build_mask(c["hq"], seqs, c["tile"], c["tile"], c["g"], c["causal"], c["p"], c["seed"] + 4,
                             True, True)
    return q.numpy(), k.numpy(), v.numpy(), seqs, mask


def _oracle_heads(q, k, v, seqs, mask, s0, s1, k0, k1):
    c = CASE
    qs, ks = q[:, s0:s1], k[:, k0:k1]
    return oracle.attention(qs, ks, v[:, k0:k1], causal=c["causal"], tile_m=c["tile"], tile_n=c["tile"],
                            g=c["g"], mask=mask[s0:s1],
                            q_quant=oracle.quantize_tiles(qs, seqs, c["tile"], "q"),
                            k_quant=oracle.quantize_tiles(ks, seqs, c["tile"], "k"))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = CASE
        q, k, v, seqs, mask = _problem()
        shards = dist.head_shards(c["hq"], world)
        h0, h1 = shards[rank]
        h_cap = max(b - a for a, b in shards)
        local = torch.zeros((c["L"], h_cap, c["d"]), dtype=torch.float64)
        segs = dist.kv_segments(h0, h1, c["hq"] // c["hkv"])
        for s0, s1, k0, k1 in segs:
            local[:, s0 - h0:s1 - h0] = torch.from_numpy(_oracle_heads(q, k, v, seqs, mask, s0, s1, k0, k1))
        gathered = torch.empty((world, c["L"], h_cap, c["d"]), dtype=torch.float64)
        dist.all_gather_heads(gathered, local)
        merged = torch.empty((c["L"], c["hq"], c["d"]), dtype=torch.float64)
        for r, (a, b) in enumerate(shards):
            merged[:, a:b] = gathered[r, :, :b - a]
        out[rank] = (segs, merged.numpy())
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_head_sharded_equals_unsharded():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    c = CASE
    q, k, v, seqs, mask = _problem()
    full = _oracle_heads(q, k, v, seqs, mask, 0, c["hq"], 0, c["hkv"])
    # 6 query heads over 3 KV heads (2 per group): rank 0 holds 0..2, rank 1 holds 3..5,
    # each cutting the middle group
    assert out[0][0] == [(0, 2, 0, 1), (2, 3, 1, 2)]
    assert out[1][0] == [(3, 4, 1, 2), (4, 6, 2, 3)]
    for r in range(world):
        np.testing.assert_array_equal(out[r][1], full)      # every rank holds the whole output
    assert np.isfinite(full).all() and np.abs(full).max() > 0


# ---------------------------------------------------------------- C-ABI validation
def _merge_status(out, stride, gathered, T, Hq, d, world, h_cap, head_start):
    hs = None if head_start is None else np.ascontiguousarray(np.asarray(head_start, dtype=np.int32))
    return ops._lib().tm_merge_head_shards(out, stride, gathered, T, Hq, d, world, h_cap,
                                           None if hs is None else hs.ctypes.data, None), hs


@pytest.mark.parametrize("args", [
    dict(head_start=None),                                   # no head table
    dict(head_start=[0, 3, 5]),                              # does not end at Hq = 6
    dict(head_start=[1, 3, 6]),                              # does not start at 0
    dict(head_start=[0, 4, 6], h_cap=3),                     # a shard larger than h_cap
    dict(head_start=[0, 4, 3, 6], world=3),                  # decreasing
    dict(d=60),                                              # d not a multiple of 8
    dict(stride=6 * 64 - 8),                                 # row stride below Hq * d
    dict(stride=6 * 64 + 4),                                 # row stride not a multiple of 8
    dict(world=0, head_start=[0]),
    dict(world=65, head_start=list(range(0, 66))),
    dict(out=None),                                          # null pointers with rows to copy
    dict(out=0x1008),                                        # misaligned output
])
def test_merge_rejects_bad_arguments_before_any_cuda_call(args):
    a = dict(out=0x1000, stride=6 * 64, gathered=0x2000, T=10, Hq=6, d=64, world=2, h_cap=3,
             head_start=[0, 3, 6])
    a.update(args)
    if a["world"] == 65:
        a["Hq"] = 65
        a["stride"] = 65 * 64
    st, _ = _merge_status(None if a["out"] is None else ctypes.c_void_p(a["out"]), a["stride"],
                          ctypes.c_void_p(a["gathered"]), a["T"], a["Hq"], a["d"], a["world"], a["h_cap"],
                          a["head_start"])
    assert st == ops.TM_ERR_INVALID_ARG


def test_merge_of_zero_rows_is_a_no_op():
    st, _ = _merge_status(None, 6 * 64, None, 0, 6, 64, 2, 3, [0, 3, 6])
    assert st == ops.TM_OK
