"""Seeded synthetic inputs for tile-routed attention.

This module only draws inputs: it holds none of the attention, quantisation
or routing arithmetic of the method, and it imports neither the CUDA binding
nor the CPU oracle, so both sides can be fed identical bits from it.

Every tensor is drawn on the CPU with ``torch.Generator().manual_seed(s)`` as
fp32, shaped and scaled in fp32, then rounded once to fp16 (round to nearest
even).  Seed convention for a workload with base seed s: Q = s, K = s + 1,
V = s + 2, outlier channels = s + 3, routing mask = s + 4, sequence lengths
= s + 5.

Workload shapes follow the pages' benchmark tables: the MLX fused-SDPA table
(B = 1, fp16, qsl/ksl in {512, 1024, 2048, 4096}, hdim in {64, 128},
n_qh/n_kvh pairs (32,32), (32,8), (16,2)) and the TileMix abstract's
long-context prefill with GQA, variable-length batches and INT8 K/V caches.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn_f16(shape, seed, scale=1.0):
    """N(0, scale^2) fp32 draws rounded once to fp16."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.float16)


def outlier_channels(hkv, d, seed, n=4):
    """n distinct channel indices per KV head, int64 [hkv, n]."""
    g = _gen(seed)
    return torch.stack([torch.randperm(d, generator=g)[:n] for _ in range(hkv)])


def qk_with_outliers(Tq, Tk, hq, hkv, d, seed, factor=20.0, n=4):
    """Q [Tq, hq, d] and K [Tk, hkv, d] ~ N(0, 1), with n seeded channels per
    KV head multiplied by ``factor`` in K[:, hk] and in every query head of
    that KV head's group (hq // hkv consecutive heads).  Scaling happens in
    fp32 before the single rounding to fp16."""
    q = torch.randn(Tq, hq, d, generator=_gen(seed), dtype=torch.float32)
    k = torch.randn(Tk, hkv, d, generator=_gen(seed + 1), dtype=torch.float32)
    ch = outlier_channels(hkv, d, seed + 3, n)
    grp = hq // hkv
    for hk in range(hkv):
        idx = ch[hk]
        k[:, hk, idx] *= factor
        q[:, hk * grp:(hk + 1) * grp, idx] *= factor
    return q.to(torch.float16), k.to(torch.float16), ch


def qk_with_token_outliers(Tq, Tk, hq, hkv, d, seed, factor=20.0, frac=0.002):
    """Q [Tq, hq, d] and K [Tk, hkv, d] ~ N(0, 1), with a seeded fraction of
    key tokens (the same tokens for every KV head) multiplied by ``factor`` in
    all channels, in fp32 before the single rounding to fp16: outliers that
    sit in a few key tiles rather than in every tile.  Returns (q, k, the
    outlier token indices)."""
    q = torch.randn(Tq, hq, d, generator=_gen(seed), dtype=torch.float32)
    k = torch.randn(Tk, hkv, d, generator=_gen(seed + 1), dtype=torch.float32)
    n = max(1, int(round(frac * Tk)))
    tok = torch.randperm(Tk, generator=_gen(seed + 3))[:n].sort().values
    k[tok] *= factor
    return q.to(torch.float16), k.to(torch.float16), tok


def varlen_lengths(batch, lo, hi, seed):
    """batch integer lengths ~ U[lo, hi] (inclusive) and cu_seqlens int32."""
    lens = torch.randint(lo, hi + 1, (batch,), generator=_gen(seed), dtype=torch.int64)
    cu = torch.zeros(batch + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    return lens, cu


def lossless_qk(seqs_q, seqs_k, Tq, Tk, hq, hkv, d, tile_m, tile_n, seed):
    """Inputs whose per-tile INT8 codes are exact.

    Every value is an integer in [-127, 127] times 2^-6, and each (tile, head)
    block holds at least one +-127 * 2^-6, so the tile absmax is exactly
    127 * 2^-6.  ``seqs_q`` / ``seqs_k`` are lists of (start, length) that
    say where the tiles restart.
    """
    def draw(T, H, seqs, tile, s):
        g = _gen(s)
        x = torch.randint(-127, 128, (T, H, d), generator=g, dtype=torch.int32).to(torch.float32)
        for start, length in seqs:
            for r0 in range(0, length, tile):
                rows = min(tile, length - r0)
                for h in range(H):
                    r = int(torch.randint(0, rows, (1,), generator=g))
                    c = int(torch.randint(0, d, (1,), generator=g))
                    sign = 1.0 if int(torch.randint(0, 2, (1,), generator=g)) else -1.0
                    x[start + r0 + r, h, c] = 127.0 * sign
        return (x * 2.0 ** -6).to(torch.float16)
    return draw(Tq, hq, seqs_q, tile_m, seed), draw(Tk, hkv, seqs_k, tile_n, seed + 1)


def int8_kv_cache(x16):
    """Per-(token, head) INT8 cache of an fp16 tensor [T, H, d]: the caller's
    cache format, produced here as input data.  scale = fp16_rn(amax / 127)
    over the token's d values; code = clamp(rne(x / scale), -127, 127) with x
    and scale in fp32; a zero row gives scale 0 and codes 0."""
    x = x16.to(torch.float32)
    amax = x.abs().amax(dim=-1)
    scale16 = (amax / 127.0).to(torch.float16)
    s = scale16.to(torch.float32)
    safe = torch.where(s > 0, s, torch.ones_like(s))
    codes = torch.round(x / safe[..., None]).clamp_(-127, 127)
    codes = torch.where(s[..., None] > 0, codes, torch.zeros_like(codes)).to(torch.int8)
    return codes, scale16


@dataclass
class Workload:
    """One seeded attention problem (CPU tensors)."""
    name: str
    q: torch.Tensor
    k: torch.Tensor | None
    v: torch.Tensor | None
    hq: int
    hkv: int
    d: int
    causal: bool
    tile_m: int
    tile_n: int
    g: int
    p: float | None                      # Bernoulli parameter of the mask (None: all FP16)
    mask_seed: int = 0
    force_diag: bool = False
    force_sink: bool = False
    cu_seqlens: torch.Tensor | None = None
    lens: torch.Tensor | None = None
    kv_cache: tuple | None = None        # (k_codes, k_scale16, v_codes, v_scale16)
    extra: dict = field(default_factory=dict)
    cu_seqlens_k: torch.Tensor | None = None   # key offsets when they differ (prefix-cached prefill)
    lens_k: torch.Tensor | None = None

    @property
    def Lq(self):
        return int(self.q.shape[0])

    @property
    def Lk(self):
        return int((self.k if self.k is not None else self.kv_cache[0]).shape[0])

    @property
    def max_seqlen(self):
        if self.lens is not None:
            return int(self.lens.max())
        return max(self.Lq, self.Lk)

    @property
    def max_seqlen_k(self):
        return None if self.lens_k is None else int(self.lens_k.max())


def tiny(seed=0, p=None):
    """B=1, Hq=2, Hkv=1, L=256, d=64, non-causal, tiles 64x64, g=1."""
    L, hq, hkv, d = 256, 2, 1, 64
    return Workload("tiny", randn_f16((L, hq, d), seed), randn_f16((L, hkv, d), seed + 1),
                    randn_f16((L, hkv, d), seed + 2), hq, hkv, d, False, 64, 64, 1, p,
                    mask_seed=seed + 4)


def mlx_shape(Lq, Lk, d, hq, hkv, causal, seed=0):
    """MLX-table shape, all-FP16 routing, tiles 128x128."""
    return Workload(f"mlx_q{Lq}_k{Lk}_d{d}_h{hq}x{hkv}_c{int(causal)}",
                    randn_f16((Lq, hq, d), seed), randn_f16((Lk, hkv, d), seed + 1),
                    randn_f16((Lk, hkv, d), seed + 2), hq, hkv, d, causal, 128, 128, 1, None)


MLX_SHAPES = [(L, L, d, hq, hkv) for L in (1024, 2048, 4096) for d in (64, 128)
              for (hq, hkv) in ((32, 32), (32, 8), (16, 2))] + \
             [(512, 4096, d, hq, hkv) for d in (64, 128) for (hq, hkv) in ((32, 32), (32, 8), (16, 2))]


def routing_sweep(p, L=16384, hq=32, hkv=8, d=128, seed=0):
    """Causal, tiles 128x128, g=4, outlier channels x20, diagonal and sink
    groups forced FP16, Bernoulli(p) INT8 mask."""
    q, k, ch = qk_with_outliers(L, L, hq, hkv, d, seed)
    v = randn_f16((L, hkv, d), seed + 2)
    return Workload(f"sweep_L{L}_p{p}", q, k, v, hq, hkv, d, True, 128, 128, 4, p,
                    mask_seed=seed + 4, force_diag=True, force_sink=True,
                    extra={"outlier_channels": ch})


def routing_sweep_token_outliers(p, L=16384, hq=32, hkv=8, d=128, seed=0, frac=0.002):
    """The routing-sweep shape with token-localised key outliers
    (qk_with_token_outliers) instead of outlier channels."""
    q, k, tok = qk_with_token_outliers(L, L, hq, hkv, d, seed, frac=frac)
    v = randn_f16((L, hkv, d), seed + 2)
    return Workload(f"sweep_tokout_L{L}_p{p}", q, k, v, hq, hkv, d, True, 128, 128, 4, p,
                    mask_seed=seed + 4, force_diag=True, force_sink=True,
                    extra={"outlier_tokens": int(tok.numel())})


def varlen_int8_cache(batch=8, lo=1024, hi=8192, hq=32, hkv=4, d=128, p=0.75, seed=0):
    """Packed variable-length causal batch with an INT8 K/V cache (per token
    and head fp16 scales), Q fp16, g=4, Bernoulli(p) mask, diagonal and sink
    groups forced FP16."""
    lens, cu = varlen_lengths(batch, lo, hi, seed + 5)
    T = int(cu[-1])
    q = randn_f16((T, hq, d), seed)
    k = randn_f16((T, hkv, d), seed + 1)
    v = randn_f16((T, hkv, d), seed + 2)
    kc, ks = int8_kv_cache(k)
    vc, vs = int8_kv_cache(v)
    return Workload(f"varlen_cache_b{batch}", q, None, None, hq, hkv, d, True, 128, 128, 4, p,
                    mask_seed=seed + 4, force_diag=True, force_sink=True,
                    cu_seqlens=cu, lens=lens, kv_cache=(kc, ks, vc, vs))


def prefix_int8_cache(batch=8, lo=256, hi=2048, prefix_hi=8192, hq=32, hkv=4, d=128, p=0.75, seed=0):
    """Prefix-cached prefill over an INT8 K/V cache: sequence b has lq ~
    U[lo, hi] new query tokens and a cached prefix of U[0, prefix_hi] tokens,
    so lk = prefix + lq keys (cu_seqlens_k); causal (bottom-right), g=4,
    Bernoulli(p) mask, diagonal and sink groups forced FP16."""
    lq, cu = varlen_lengths(batch, lo, hi, seed + 5)
    pre, _ = varlen_lengths(batch, 0, prefix_hi, seed + 6)
    lk = lq + pre
    cu_k = torch.zeros(batch + 1, dtype=torch.int32)
    cu_k[1:] = torch.cumsum(lk, 0).to(torch.int32)
    q = randn_f16((int(cu[-1]), hq, d), seed)
    k = randn_f16((int(cu_k[-1]), hkv, d), seed + 1)
    v = randn_f16((int(cu_k[-1]), hkv, d), seed + 2)
    kc, ks = int8_kv_cache(k)
    vc, vs = int8_kv_cache(v)
    return Workload(f"prefix_cache_b{batch}", q, None, None, hq, hkv, d, True, 128, 128, 4, p,
                    mask_seed=seed + 4, force_diag=True, force_sink=True,
                    cu_seqlens=cu, lens=lq, kv_cache=(kc, ks, vc, vs), cu_seqlens_k=cu_k, lens_k=lk)


def long_context(L=65536, hq=28, hkv=4, d=128, p=0.5, seed=0):
    """Causal, tiles 128x128, g=8, outliers as in the routing sweep, Bernoulli(p)
    mask with diagonal and sink groups forced FP16."""
    q, k, ch = qk_with_outliers(L, L, hq, hkv, d, seed)
    v = randn_f16((L, hkv, d), seed + 2)
    return Workload(f"long_L{L}", q, k, v, hq, hkv, d, True, 128, 128, 8, p,
                    mask_seed=seed + 4, force_diag=True, force_sink=True,
                    extra={"outlier_channels": ch})
