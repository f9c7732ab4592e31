"""The bench line's parity sample (bench.cpu_baseline) on CPU: fed an output
equal to the oracle's (rounded to fp16, as the kernels write it) it passes
within the fp16 rounding of the output; with one planted error in a sampled
row it reports that error.  The GPU output is stood in for by the oracle's
own output here, so no GPU is involved."""

import numpy as np
import torch

import bench
import oracle
from mixed_precision_attention_tm_b200 import inputs


def _oracle_out(w):
    seqs = oracle.seq_table(w.Lq, w.Lk)
    kw = dict(causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g)
    if w.p is not None:
        q, k = w.q.numpy(), w.k.numpy()
        kw.update(mask=oracle.build_mask(w.hq, seqs, w.tile_m, w.tile_n, w.g, w.causal, w.p, w.mask_seed,
                                         w.force_diag, w.force_sink),
                  q_quant=oracle.quantize_tiles(q, seqs, w.tile_m, "q"),
                  k_quant=oracle.quantize_tiles(k, seqs, w.tile_n, "k"))
    return oracle.attention(w.q.numpy(), w.k.numpy(), w.v.numpy(), **kw)


def test_parity_sample_passes_on_exact_output_and_reports_a_planted_error():
    w = inputs.tiny(seed=0, p=0.5)
    ref = _oracle_out(w)
    w.extra["gpu_out"] = torch.from_numpy(ref.astype(np.float16))
    base, parity = bench.cpu_baseline(w, 0.5)
    assert base["kind"] == "oracle" and base["value"] > 0
    assert parity["pass"] and parity["rows_compared"] > 0
    assert parity["max_abs_err"] <= 2.0 ** -11 * float(np.abs(ref).max())   # fp16 rounding only
    bad = ref.astype(np.float16)
    bad[70, 1, 5] += np.float16(0.25)           # row 70: second 64-row tile, head 1
    w.extra["gpu_out"] = torch.from_numpy(bad)
    _, parity = bench.cpu_baseline(w, 0.5)
    assert not parity["pass"] and parity["max_abs_err"] >= 0.24


def test_no_gpu_output_gives_no_parity_entry():
    w = inputs.tiny(seed=1)
    base, parity = bench.cpu_baseline(w, 0.2)
    assert parity is None and base["value"] > 0
