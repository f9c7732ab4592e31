"""GPU parity at the benchmark configurations' full sizes, through the same
calls bench.py times: the whole output is computed on the GPU, and sampled
query rows (tile boundaries plus seeded random rows, every head) are compared
with the fp64 oracle, which evaluates those rows one by one.  Routing bits,
INT8 codes and tile scales are compared in full (bit-exact).

With TM_PARITY_REPORT set to a file path, one JSON line per configuration
(rows compared, max-abs error, bound) is appended to that file.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL, max_err, oracle_mask, run_gpu, run_oracle, seqs_of
from mixed_precision_attention_tm_b200 import inputs, ops

pytestmark = pytest.mark.gpu

_REPORT = []


@pytest.fixture(scope="module", autouse=True)
def _parity_report():
    yield
    path = os.environ.get("TM_PARITY_REPORT")
    if path and _REPORT:
        with open(path, "a") as f:
            for r in _REPORT:
                f.write(json.dumps(r) + "\n")


def _record(w, rows, err, exact):
    _REPORT.append({"workload": w.name, "heads": w.hq, "rows_compared": rows, "max_abs_err": err,
                    "bound": TOL, "codes_scales_mask": exact})


def _sample_rows(seqs, tile, n_random, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for (qs, lq, _ks, _lk) in seqs:
        if lq == 0:
            continue
        rows.update([qs, qs + lq - 1])
        for r0 in range(0, lq, tile * 16):       # first and last row of every 16th tile
            rows.update([qs + r0, qs + min(lq, r0 + tile) - 1])
        rows.update(int(x) for x in rng.integers(qs, qs + lq, max(1, n_random // len(seqs))))
    return sorted(rows)


def _check(w, n_random=48):
    out, m, quant = run_gpu(w)
    assert torch.isfinite(out).all()
    seqs, _ = seqs_of(w)
    mask_u32 = None if m is None else m.numpy().view(np.uint32)
    exact = "no mask"
    if mask_u32 is not None:
        assert np.array_equal(mask_u32, oracle_mask(w))
        rq = oracle.quantize_tiles(w.q.numpy(), seqs, w.tile_m, "q")
        assert np.array_equal(quant[1].numpy(), rq[1]) and np.array_equal(quant[0].numpy(), rq[0])
        if quant[2] is not None:
            rk = oracle.quantize_tiles(w.k.numpy(), seqs, w.tile_n, "k")
            assert np.array_equal(quant[3].numpy(), rk[1]) and np.array_equal(quant[2].numpy(), rk[0])
        exact = "bit-exact"
    rows = _sample_rows(seqs, w.tile_m, n_random, 17)
    ref = run_oracle(w, mask_u32, rows=rows)
    err = max_err(out, ref, rows=rows)
    _record(w, f"{len(rows)} sampled rows x all heads", err, exact)
    assert err <= TOL, f"{w.name}: max abs err {err} over {len(rows)} rows"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk,d,hq,hkv", inputs.MLX_SHAPES)
def test_mlx_shapes_full_size(Lq, Lk, d, hq, hkv, causal):
    """All 48 runs of the MLX-shaped configuration (24 shapes of the MLX PR
    "Nax Refactor" attention tables, causal and not), each at its own size,
    through the library's automatic kernel choice as bench.py times them."""
    _check(inputs.mlx_shape(Lq, Lk, d, hq, hkv, causal), n_random=32)


@pytest.mark.parametrize("p", [0.0, 0.75, 1.0])
def test_routing_sweep_full_size(p):
    _check(inputs.routing_sweep(p))


def test_varlen_int8_cache_full_size():
    _check(inputs.varlen_int8_cache(), n_random=64)


def _check_plan(w, n_random=48):
    """Full size through the prefill plan exactly as bench.py builds and times
    it (for an INT8 cache: the cache expanded into the plan's workspace)."""
    from mixed_precision_attention_tm_b200.api import TileMixPrefill
    pl = TileMixPrefill(w.Lq, w.Lk, w.hq, w.hkv, w.d, causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g,
                        p=w.p, seed=w.mask_seed, force_diag=w.force_diag, force_sink=w.force_sink,
                        cu_seqlens=w.cu_seqlens, int8_cache=w.kv_cache is not None, cu_seqlens_k=w.cu_seqlens_k)
    pl.load(w.q, w.k, w.v, w.kv_cache)
    out = pl.run().cpu()
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    assert torch.isfinite(out).all()
    cu = None if w.cu_seqlens is None else w.cu_seqlens.tolist()
    ck = None if w.cu_seqlens_k is None else w.cu_seqlens_k.tolist()
    seqs = oracle.seq_table(w.Lq, w.Lk, cu, ck)
    mask_u32 = pl.bitmask.cpu().numpy().view(np.uint32)
    assert np.array_equal(mask_u32, oracle.build_mask(w.hq, seqs, w.tile_m, w.tile_n, w.g, w.causal, w.p,
                                                      w.mask_seed, w.force_diag, w.force_sink))
    rq = oracle.quantize_tiles(w.q.numpy(), seqs, w.tile_m, "q")
    assert np.array_equal(pl.q_quant[1].cpu().numpy(), rq[1]) and np.array_equal(pl.q_quant[0].cpu().numpy(), rq[0])
    rows = _sample_rows(seqs, w.tile_m, n_random, 17)
    ref = oracle.attention(w.q.numpy(), kv_cache=tuple(t.numpy() for t in w.kv_cache), cu_seqlens=cu,
                           cu_seqlens_k=ck, causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g,
                           mask=mask_u32, q_quant=rq, rows=rows)
    err = max_err(out, ref, rows=rows)
    _record(w, f"{len(rows)} sampled rows x all heads (plan, cache workspace)", err, "bit-exact")
    assert err <= TOL, f"{w.name}: max abs err {err} over {len(rows)} rows"


def test_varlen_int8_cache_full_size_through_the_plan():
    _check_plan(inputs.varlen_int8_cache(), n_random=64)


def test_prefix_int8_cache_full_size_through_the_plan():
    _check_plan(inputs.prefix_int8_cache(), n_random=64)


def test_long_context_full_size():
    _check(inputs.long_context(), n_random=24)


def test_tiny_config_both_runs():
    for p in (None, 0.5):
        w = inputs.tiny(seed=0, p=p)
        out, m, _ = run_gpu(w)
        if m is not None:
            assert np.array_equal(m.numpy().view(np.uint32), oracle_mask(w))
        ref = run_oracle(w, None if m is None else m.numpy().view(np.uint32))
        err = max_err(out, ref)
        _record(w, "all rows", err, "no mask" if m is None else "mask bit-exact")
        assert err <= TOL
