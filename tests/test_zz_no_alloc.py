"""GPU test of tm_attn_fwd_routed_noalloc, the routed prefill entry point for
callers that cannot allocate device memory (for instance engines that keep
all device memory in their own pools, or deployments that forbid cudaMalloc
after start-up).  It keeps the INT8 codes, tile scales and routing mask in a
fixed library-owned device array; its output must match the regular path
(tm_quantize_qk + tm_build_mask + tm_attn_fwd with caller-allocated buffers)
within the parity tolerance, on two calls in a row that reuse the array.

Collected last on purpose: a run that stops at the first failure has already
run every other test.
"""

import pytest
import torch

from gpu_helpers import TOL
from mixed_precision_attention_tm_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def _regular(q, k, v, tm, tn, g, causal, p, seed, fd, fs):
    qc, qs, kc, ks = ops.quantize_qk(q, k, tile_m=tm, tile_n=tn)
    m = ops.build_mask(q.shape[1], tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed, force_diag=fd,
                       force_sink=fs, Lq=q.shape[0], Lk=k.shape[0], device=q.device)
    return ops.attn_fwd(q, k, v, tile_m=tm, tile_n=tn, g=g, causal=causal, bitmask=m, q_quant=(qc, qs),
                        k_quant=(kc, ks))


CALLS = [
    # (Lq, Lk, Hq, Hkv, d, tile_m, tile_n, g, causal, p, seed, force_diag, force_sink)
    (1024, 1024, 8, 2, 128, 128, 128, 2, True, 0.5, 11, True, True),
    (700, 900, 4, 1, 64, 64, 64, 1, False, 0.75, 12, False, True),
]


def test_noalloc_matches_regular_path_on_consecutive_calls():
    # The first call is the larger one, so the second reuses an array that
    # still holds longer codes, scales and mask rows from the first.
    for i, (Lq, Lk, hq, hkv, d, tm, tn, g, causal, p, seed, fd, fs) in enumerate(CALLS):
        q = inputs.randn_f16((Lq, hq, d), seed).cuda()
        k = inputs.randn_f16((Lk, hkv, d), seed + 1).cuda()
        v = inputs.randn_f16((Lk, hkv, d), seed + 2).cuda()
        got = ops.attn_fwd_routed_noalloc(q, k, v, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed,
                                          force_diag=fd, force_sink=fs)
        ref = _regular(q, k, v, tm, tn, g, causal, p, seed, fd, fs)
        torch.cuda.synchronize()
        assert ops.get_device_error() == ops.TM_OK
        # the same kernels on the same inputs: the outputs are bit-identical
        assert torch.equal(got, ref), f"call {i}: max abs difference {(got.float() - ref.float()).abs().max().item()}"


def test_noalloc_call_leaves_device_memory_unchanged():
    Lq, Lk, hq, hkv, d, tm, tn, g, causal, p, seed, fd, fs = CALLS[0]
    q = inputs.randn_f16((Lq, hq, d), seed).cuda()
    k = inputs.randn_f16((Lk, hkv, d), seed + 1).cuda()
    v = inputs.randn_f16((Lk, hkv, d), seed + 2).cuda()
    out = torch.empty_like(q)
    kw = dict(out=out, tile_m=tm, tile_n=tn, g=g, causal=causal, p=p, seed=seed, force_diag=fd, force_sink=fs)
    ops.attn_fwd_routed_noalloc(q, k, v, **kw)   # first call on the device: module and symbol set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    ops.attn_fwd_routed_noalloc(q, k, v, **kw)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    assert torch.equal(out, _regular(q, k, v, tm, tn, g, causal, p, seed, fd, fs))


def test_noalloc_rejects_problems_beyond_the_array():
    # 32 MiB of scratch cannot hold the codes of 16384 x 32 x 128 queries
    q = torch.empty((16384, 32, 128), dtype=torch.float16, device="cuda")
    k = torch.empty((16384, 8, 128), dtype=torch.float16, device="cuda")
    v = torch.empty_like(k)
    with pytest.raises(ops.TmError) as e:
        ops.attn_fwd_routed_noalloc(q, k, v, causal=True, p=0.5)
    assert e.value.status == ops.TM_ERR_UNSUPPORTED
