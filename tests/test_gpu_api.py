"""GPU checks of the public plan API: the pipelined host runner (copies of
neighbouring steps overlapped with compute) returns, for every step, exactly
the output of a direct device call on the same inputs."""

import pytest
import torch

from mixed_precision_attention_tm_b200 import inputs
from mixed_precision_attention_tm_b200.api import HostPipeline, TileMixPrefill

pytestmark = pytest.mark.gpu


def test_host_pipeline_matches_direct_steps():
    L, hq, hkv, d = 1024, 4, 2, 128
    batches = []
    for s in range(3):
        q, k, _ = inputs.qk_with_outliers(L, L, hq, hkv, d, seed=10 * s)
        v = inputs.randn_f16((L, hkv, d), 10 * s + 2)
        batches.append((q.pin_memory(), k.pin_memory(), v.pin_memory(), None))
    kw = dict(causal=True, tile_m=128, tile_n=128, g=2, p=0.5, seed=3, force_diag=True, force_sink=True)
    pipe = HostPipeline(L, L, hq, hkv, d, **kw)
    outs = [torch.empty((L, hq, d), dtype=torch.float16, pin_memory=True) for _ in range(5)]
    steps = [batches[i % 3] for i in range(5)]
    last = pipe.run(steps, outs)
    last.synchronize()
    direct = TileMixPrefill(L, L, hq, hkv, d, **kw)
    for i, (q, k, v, _) in enumerate(steps):
        direct.load(q.cuda(), k.cuda(), v.cuda())
        ref = direct.run().cpu()
        assert torch.equal(outs[i], ref), i
