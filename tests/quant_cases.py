"""Constructed inputs for the INT8 tile quantiser's rounding boundaries (test
infrastructure).  With s = fl32(amax / 127), a code is rne(fl32(x / s)); the
cases below put x / s exactly on a half-integer (power-of-two scales) or
within 2^-13 of one, where an implementation that forms x / s any other way
than one IEEE division is most likely to round differently."""

import numpy as np


def all_f16_up_to(amax):
    """Every finite fp16 value in [-amax, amax]."""
    bits = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)
    pos = bits[bits.astype(np.float32) <= np.float32(amax)]
    return np.concatenate([pos, -pos])


def near_tie_values(amax, limit=2.0 ** -13):
    """fp16 values x in [-amax, amax] whose exact quotient x / s, with
    s = fl32(amax / 127), lies within `limit` of a half-integer."""
    s = np.float64(np.float32(np.float32(amax) / np.float32(127.0)))
    x = all_f16_up_to(amax)
    q = x.astype(np.float64) / s
    frac = np.abs(q - np.floor(q) - 0.5)
    return x[frac <= limit]


def tie_tile(rows, d, amax, seed):
    """A rows x d fp16 tile holding amax once and otherwise near-tie values of
    that amax (cycled, shuffled by seed)."""
    v = near_tie_values(amax)
    rng = np.random.default_rng(seed)
    if v.size == 0:
        v = np.array([np.float16(0.0)])
    t = rng.permutation(np.resize(v, rows * d)).astype(np.float16).reshape(rows, d)
    t[rows // 2, d // 3] = np.float16(amax)
    return t


# fp16 amax values: powers-of-two multiples of 127 (exact scales, exact
# ties), values just off them, and assorted others.
AMAXES = [127.0, 1.984375, 0.2480469, 127.0625, 2.0, 3.140625, 0.0117, 5.96e-6, 1000.0, 60000.0, 7.5, 0.5]
