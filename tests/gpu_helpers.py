"""Shared helpers of the GPU parity tests: run one workload through the C-ABI
(ops) and through the oracle on the same seeded inputs."""

import numpy as np
import torch

import oracle
from mixed_precision_attention_tm_b200 import ops

TOL = 3e-3   # max-abs output error vs the fp64 oracle (fp16 output, unit-variance inputs)


def seqs_of(w):
    cu = None if w.cu_seqlens is None else w.cu_seqlens.tolist()
    return oracle.seq_table(w.Lq, w.Lk, cu), cu


def run_gpu(w, mask=None, quant=None):
    """Quantise (when routed), build the device mask (when w.p is not None and
    no mask is given) and run the fused kernel.  Returns (out fp16 CPU, mask
    CPU int32 or None, (qc, qs, kc, ks) CPU or None)."""
    dev = "cuda"
    q = w.q.to(dev)
    cu = None if w.cu_seqlens is None else w.cu_seqlens.to(dev)
    kv = None
    if w.kv_cache is not None:
        kv = tuple(t.to(dev) for t in w.kv_cache)
        k = v = None
    else:
        k, v = w.k.to(dev), w.v.to(dev)
    qq = kq = None
    m = None
    if w.p is not None or mask is not None:
        qc, qs, kc, ks = ops.quantize_qk(q, k, tile_m=w.tile_m, tile_n=w.tile_n, cu_seqlens=cu,
                                         max_seqlen=w.max_seqlen if cu is not None else None)
        qq, kq = (qc, qs), (None if k is None else (kc, ks))
        if mask is None:
            m = ops.build_mask(w.hq, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g, causal=w.causal, p=w.p,
                               seed=w.mask_seed, force_diag=w.force_diag, force_sink=w.force_sink,
                               Lq=w.Lq, Lk=w.Lk, cu_seqlens=cu, max_seqlen=w.max_seqlen)
        else:
            m = torch.as_tensor(np.asarray(mask).view(np.int32)).to(dev)
    out = ops.attn_fwd(q, k, v, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g, causal=w.causal, bitmask=m,
                       q_quant=qq, k_quant=kq, kv_cache=kv, cu_seqlens=cu,
                       max_seqlen=w.max_seqlen if cu is not None else None)
    torch.cuda.synchronize()
    assert ops.get_device_error() == ops.TM_OK
    quant = None
    if qq is not None:
        quant = (qq[0].cpu(), qq[1].cpu(), None if kq is None else kq[0].cpu(), None if kq is None else kq[1].cpu())
    return out.cpu(), (None if m is None else m.cpu()), quant


def run_oracle(w, mask_u32=None, rows=None):
    seqs, cu = seqs_of(w)
    q = w.q.numpy()
    kw = dict(cu_seqlens=cu, causal=w.causal, tile_m=w.tile_m, tile_n=w.tile_n, g=w.g, rows=rows)
    if w.kv_cache is not None:
        kw["kv_cache"] = tuple(t.numpy() for t in w.kv_cache)
        k = v = None
    else:
        k, v = w.k.numpy(), w.v.numpy()
    if mask_u32 is not None:
        kw["mask"] = mask_u32
        kw["q_quant"] = oracle.quantize_tiles(q, seqs, w.tile_m, "q")
        if w.kv_cache is None:
            kw["k_quant"] = oracle.quantize_tiles(k, seqs, w.tile_n, "k")
    return oracle.attention(q, k, v, **kw)


def oracle_mask(w):
    seqs, _ = seqs_of(w)
    return oracle.build_mask(w.hq, seqs, w.tile_m, w.tile_n, w.g, w.causal, w.p, w.mask_seed,
                             w.force_diag, w.force_sink)


def max_err(out_gpu, ref, rows=None):
    o = out_gpu.to(torch.float64).numpy()
    if rows is not None:
        o, ref = o[rows], ref[rows]
    return float(np.max(np.abs(o - ref))) if o.size else 0.0
