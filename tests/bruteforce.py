"""Scalar pure-Python restatement of tile-routed attention, for tiny inputs.

Written independently of ``oracle/`` (no shared helpers): plain loops over
rows, keys and channels, Python floats (binary64) for the attention, and the
fp32 steps of the quantiser emulated with ``struct`` round trips.  It pins
the vectorised oracle on inputs of a few rows.

Source of the rules: TileMix (Lattice paper page), abstract -- score tiles,
one routing bit per (query tile, group of g key tiles), FP16 or INT8 score per
group, shared softmax, GQA, varlen, INT8 K/V cache; MLX PR "Nax Refactor"
attention tables -- causal fp16 SDPA with bottom-right alignment.
"""

import math
import struct


def f32(x):
    """Round a binary64 value to the nearest binary32 (ties to even)."""
    return struct.unpack("f", struct.pack("f", float(x)))[0]


def quant_block(vals):
    """vals: list of floats exactly representable in fp16.  Returns (scale,
    codes).  fl32(a / b) is computed as f32(a / b) in binary64: the quotient
    of two binary32 numbers rounded to 53 bits and then to 24 bits equals the
    directly rounded quotient (53 >= 2 * 24 + 2)."""
    amax = max((abs(v) for v in vals), default=0.0)
    s = f32(amax / 127.0)
    if s == 0.0:
        return 0.0, [0] * len(vals)
    codes = []
    for v in vals:
        r = round(f32(v / s))            # Python round: ties to even
        codes.append(max(-127, min(127, int(r))))
    return s, codes


def brute_attention(q, k, v, Hq, Hkv, d, causal, tile_m, tile_n, g, mask_bits=None,
                    cu=None, cache=None):
    """q: nested list [Tq][Hq][d] of floats; k, v: [Tk][Hkv][d] (or cache =
    (kc, ks, vc, vs) with kc [Tk][Hkv][d] ints and ks [Tk][Hkv] floats, the
    fp16 view being f16(code * scale) supplied by the caller as k, v).
    mask_bits(h, q_tile_global, group) -> 0/1 or None for all FP16.
    Returns [Tq][Hq][d] floats."""
    Tq = len(q)
    Tk = len(k)
    if cu is None:
        seqs = [(0, Tq, 0, Tk)]
    else:
        seqs = [(cu[b], cu[b + 1] - cu[b], cu[b], cu[b + 1] - cu[b]) for b in range(len(cu) - 1)]
    sigma = 1.0 / math.sqrt(d)
    out = [[[0.0] * d for _ in range(Hq)] for _ in range(Tq)]

    # quantise (per sequence, per tile, per head)
    qcode = {}
    qscale = {}
    kcode = {}
    kscale = {}
    qt_base = 0
    kt_base = 0
    bases = []
    for (qs, lq, ks, lk) in seqs:
        bases.append((qt_base, kt_base))
        nqt = (lq + tile_m - 1) // tile_m
        nkt = (lk + tile_n - 1) // tile_n
        for I in range(nqt):
            for h in range(Hq):
                rows = range(qs + I * tile_m, qs + min(lq, (I + 1) * tile_m))
                vals = [q[r][h][c] for r in rows for c in range(d)]
                s, cs = quant_block(vals)
                qscale[(h, qt_base + I)] = s
                for n, (r, c) in enumerate((r, c) for r in rows for c in range(d)):
                    qcode[(r, h, c)] = cs[n]
        if cache is None:
            for J in range(nkt):
                for h in range(Hkv):
                    rows = range(ks + J * tile_n, ks + min(lk, (J + 1) * tile_n))
                    vals = [k[r][h][c] for r in rows for c in range(d)]
                    s, cs = quant_block(vals)
                    kscale[(h, kt_base + J)] = s
                    for n, (r, c) in enumerate((r, c) for r in rows for c in range(d)):
                        kcode[(r, h, c)] = cs[n]
        qt_base += nqt
        kt_base += nkt

    for b, (qs, lq, ks, lk) in enumerate(seqs):
        qb, kb = bases[b]
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(lq):
                I = i // tile_m
                scores = []
                for j in range(lk):
                    if causal and j > i + lk - lq:
                        continue
                    J = j // tile_n
                    G = J // g
                    int8 = mask_bits is not None and mask_bits(h, qb + I, G)
                    if int8:
                        acc = 0
                        for c in range(d):
                            if cache is None:
                                ck = kcode[(ks + j, hk, c)]
                            else:
                                ck = cache[0][ks + j][hk][c]
                            acc += qcode[(qs + i, h, c)] * ck
                        sk = kscale[(hk, kb + J)] if cache is None else cache[1][ks + j][hk]
                        s = sigma * qscale[(h, qb + I)] * sk * acc
                    else:
                        s = sigma * sum(q[qs + i][h][c] * k[ks + j][hk][c] for c in range(d))
                    scores.append((j, s))
                if not scores:
                    continue
                m = max(s for _, s in scores)
                w = [(j, math.exp(s - m)) for j, s in scores]
                z = sum(x for _, x in w)
                for c in range(d):
                    out[qs + i][h][c] = sum(x * v[ks + j][hk][c] for j, x in w) / z
    return out
