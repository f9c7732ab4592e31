"""World-size-2 gloo test of the benchmark's multi-rank host logic on CPU:
ranks get distinct seeds (hence distinct batches), the step time is the
maximum over ranks, and the job throughput sums all ranks' work over that
time.  No GPU and no data-path collective are involved."""

import os
import socket

import torch
import torch.multiprocessing as mp

from mixed_precision_attention_tm_b200 import dist, inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, ws = dist.world_info()
        seed = dist.rank_seed(7, r)
        q = inputs.randn_f16((8, 2, 64), seed)
        checksum = float(q.float().sum())
        dist.barrier()
        # rank r "took" 10 + 5 r ms; every rank must see the slowest
        t = dist.max_over_ranks([10.0 + 5.0 * r, float(r)])
        out[r] = (r, lr, ws, seed, checksum, t, dist.job_throughput(ws, 2e12, t[0]))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [out[r] for r in range(world)]
    assert [x[0] for x in res] == [0, 1] and all(x[2] == world for x in res)
    assert res[0][3] == 7 and res[1][3] != res[0][3]
    assert res[0][4] != res[1][4]                                  # different batches
    for x in res:
        assert x[5] == [15.0, 1.0]                                # max over ranks
        assert abs(x[6] - world * 2e12 / 15e-3 / 1e12) < 1e-9     # whole-job TFLOP/s
